// W8A8 / W4A8 ConvRot linear on CTA pairs (tcgen05 cta_group::2), for M > 128.
//
// Same arithmetic as gemm_kernel ("MOSS-Image Qwen3.5-9B text encoder, INT8
// (W8A8, ConvRot)", file table, "Matmul" row; int4 layout of "MossInt4",
// "Format"):
//   acc[m, n] = sum_k Xq[m, k] * Wq[n, k];  Y[m, n] = bf16(float(acc) * s_tok[m] * s_row[n])
//
// Two CTAs of a cluster share one 256 x 256 output tile.  Each CTA stages its
// own 128 rows of activations (A) and its own 128 rows of weights (B, half of
// the tile's N) - 32 KB per 128-byte K atom instead of the 48 KB one CTA needs
// for a 128 x 256 tile - so each SM pulls 64 B/clk at the tensor pipe's rate.
// An int8 stage holds two K atoms (64 KB, three stages): eight MMAs per stage
// wait and commit keep the single issuing thread ahead of the tensor pipe.
// One thread of the leader CTA issues
// tcgen05.mma.cta_group::2 (256 x 256 x 32 int8): the hardware reads A and B
// from both CTAs' shared memory and writes each CTA's 128 accumulator rows x
// 256 columns into that CTA's TMEM.  TMA loads never use cluster multicast:
// each CTA loads its own tiles.
//
// Roles per CTA:
//   warp 0       TMA producer (int8: completion counted on the leader's barrier)
//   warp 1       TMEM allocation (pair-wide); in the leader, the MMA issuer
//   warps 2-9    epilogue: two warps per TMEM lane quadrant, each 128 columns;
//                bf16 (or int32) rows staged in shared memory, TMA stores
//   warps 10-13  (int4 only) unpack nibbles of this CTA's weight rows
// Work split, stream-K partial tiles and their workspace protocol are those of
// gemm_kernel with a CTA pair as the unit; each CTA of the pair fixes up its
// own 128 rows of a split tile.
//
// SPLIT (int8 weights; at most one tile per cluster): clusters of four CTAs,
// two pairs per tile.  Pair 0 accumulates the first half of K, pair 1 the
// second half.  When its MMAs are complete each CTA (its stage ring drained)
// arms a 64 KB receive barrier and tells the CTA of the other pair with the
// same rows (cluster rank +/- 2).  Each CTA stages, in its own ring, the half
// of its accumulator columns that the other CTA finalises and sends it with
// one shared-to-shared bulk copy per warp; each then adds the received half to
// its own and finalises half of the tile's columns.  The partial sums cross
// the cluster's shared-memory network, not L2, and no workspace is used.
#pragma once

#include "gemm.cuh"

namespace convrot {

constexpr int PAIR_EPI_WARPS = 8;

template <bool W4>
struct Gemm2Smem {
  static constexpr int KA = gemm_katoms(W4, true, false);
  static constexpr int A_ATOM = 128 * GEMM_BK;  // this CTA's 128 rows x one 128-byte K atom
  static constexpr int B_ATOM = 128 * GEMM_BK;
  static constexpr int A_BYTES = KA * A_ATOM;
  static constexpr int B_BYTES = KA * B_ATOM;
  // int4: the packed half-width tile of each K atom (128 rows x 64 bytes)
  // lands in the upper half of that atom's B slot and is expanded in place
  static constexpr int PACKED_OFF = B_ATOM / 2;
  static constexpr int PACKED_ATOM = 128 * (GEMM_BK / 2);
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGING = PAIR_EPI_WARPS * 4096;
  static constexpr int TMEM_COLS = 512;
  __host__ __device__ static int staging_offset(int stages) { return stages * STAGE; }
  __host__ __device__ static int bar_offset(int stages) { return stages * STAGE + STAGING; }
  __host__ __device__ static int total(int stages) {
    return bar_offset(stages) + (3 * GEMM_MAX_STAGES + 8) * 8 + 128;
  }
};

constexpr int SPLIT_RECV_BYTES = 128 * 128 * 4;  // half of one CTA's accumulator columns

// One CTA per SM.  Registers are allocated per SM sub-partition (16K each, a
// CTA's warps spread over four): with 10 (14) warps, three (four) share one,
// so 168 (128) registers per thread is the most a launch can use.
template <bool W4, int EPI, bool SPLIT = false>
__global__ void __launch_bounds__(W4 ? 448 : 320) __maxnreg__(W4 ? 128 : 168)
    gemm2sm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmY, GemmArgs a) {
  using SM = Gemm2Smem<W4>;
  static_assert(!(SPLIT && W4), "the split-K cluster mode is int8 only");
  static_assert(!(SPLIT && EPI == EPI_SWIGLU), "the split-K cluster mode has no SwiGLU epilogue");
  pdl_launch_dependents();  // the grid is co-resident: dependents only take idle SMs
  constexpr int BN = 256;
  constexpr uint32_t IDESC = idesc_s8s8s32(256, BN);

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int S = a.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::bar_offset(S));
  uint64_t* empty = full + GEMM_MAX_STAGES;
  uint64_t* conv = empty + GEMM_MAX_STAGES;
  // int8: the second K atom of a stage lands on its own barrier, so the MMAs of
  // the first atom start while the second is still in flight (the int4 kernel
  // uses these barriers for its conversion hand-off instead)
  uint64_t* full_hi = conv;
  uint64_t* tmem_full = conv + GEMM_MAX_STAGES;
  uint64_t* tmem_empty = tmem_full + 2;
  uint64_t* drain = tmem_empty + 2;
  uint64_t* epi_sync = drain + 1;
  uint64_t* recv = epi_sync + 1;   // SPLIT owner: the partner's partial has landed
  uint64_t* ready = epi_sync + 2;  // SPLIT partner: the owner's stage ring is free
  uint64_t* cv_sync = epi_sync + 3;  // int4: rendezvous of the four converter warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_sync + 4);
  // Signal slots (16 bytes each; SPLIT uses the first two for `ready`).
  // int4: four 16-byte signal slots.  The partner CTA's converter warps each
  // copy 16 bytes from their own slot into the leader's, completing bytes on
  // the leader's conversion barrier: an async-proxy hand-off instead of a
  // cluster-scope release arrive, which measured ~0.8 us per stage here.
  uint8_t* sig = reinterpret_cast<uint8_t*>(conv + GEMM_MAX_STAGES + 12);
  static_assert((3 * GEMM_MAX_STAGES + 12) % 2 == 0, "16-byte aligned signal slots");
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t rank = crank & 1u;    // role in the CTA pair: 0 = leader
  const uint32_t lead = crank & ~1u;   // cluster rank of this pair's leader
  const uint32_t pq = crank >> 1;      // SPLIT: 0 = owner pair, 1 = partner pair
  const uint16_t pair_mask = static_cast<uint16_t>(0x3u << lead);
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      // int4: the leader's 4 converter warps arrive, the partner's 4 signals complete bytes
      mbar_init(&conv[s], W4 ? 4 : 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tmem_full[b], 1);
      mbar_init(&tmem_empty[b], 2 * PAIR_EPI_WARPS);  // both CTAs' epilogue warps (leader's)
    }
    mbar_init(drain, 1);
    mbar_init(epi_sync, PAIR_EPI_WARPS);
    mbar_init(recv, 1);
    mbar_init(ready, 1);
    mbar_init(cv_sync, 4);
    *abort_flag = 0;
    *last_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, SM::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers of every CTA initialised before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // operands, scales and the output may belong to the previous kernel

  Schedule sched;
  sched.init(a, pair, npairs);
  Segment seg;
  // SPLIT: cluster u takes tile u; pair pq takes half pq of its K stages
  const int cunit = static_cast<int>(blockIdx.x >> 2);
  bool split_taken = false;
  auto next_seg = [&](Segment& sg) -> bool {
    if (!SPLIT) return sched.next(sg);
    if (split_taken || cunit >= a.num_tiles) return false;
    split_taken = true;
    const int half = (a.num_kb + 1) >> 1;
    sg.tile = cunit;
    sg.kb0 = pq ? half : 0;
    sg.kb1 = pq ? a.num_kb : half;
    sg.partial = false;
    sg.slot = -1;
    return true;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // both operands stay in L2 by preference: an A tile serves every B tile
      // of its group, a B tile the group's A tiles in the same wave; the
      // streamed output is what L2 gives up first (measured at 8192 x 24576 x
      // 4096: DRAM reads 684 -> 437 MB per launch, GEMM 3 % faster)
      const uint64_t pol_a = policy_evict_last();
      const uint64_t pol_b = policy_evict_last();
      uint32_t it = 0;
      bool ok = true;
      // No L2 prefetches run ahead of the ring: each prefetch request takes
      // the same copy engine as the loads (measured without them: 8192 x
      // 24576 x 4096 697 -> 615 us, the 36-layer int4 GEMMs 8 % faster).
      while (ok && next_seg(seg)) {
        int ta, tb;
        tile_coords(a, seg.tile, ta, tb);
        const int arow = ta * 256 + static_cast<int>(rank) * 128;
        const int brow = tb * BN + static_cast<int>(rank) * 128;
        for (int kb = seg.kb0; kb < seg.kb1; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, SITE_PROD_EMPTY)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * SM::STAGE;
          if (W4) {
            // each CTA converts its own weight rows: completion on its own barrier
            mbar_arrive_expect_tx(&full[s], SM::A_BYTES + SM::KA * SM::PACKED_ATOM);
#pragma unroll
            for (int j = 0; j < SM::KA; ++j) {
              const int k0 = (kb * SM::KA + j) * GEMM_BK;
              tma_load_2d(st + j * SM::A_ATOM, &tmA, &full[s], k0, arow, pol_a);
              tma_load_2d(st + SM::A_BYTES + j * SM::B_ATOM + SM::PACKED_OFF, &tmB, &full[s], k0 / 2,
                          brow, pol_b);
            }
          } else {
            // both CTAs' tiles complete on the leader's barriers, which the leader
            // arms: atom 0 on full[s], atom 1 on full_hi[s]
            static_assert(W4 || SM::KA == 2, "int8 pair stages hold two K atoms");
            constexpr uint32_t ATOM_TX = 2u * (SM::A_ATOM + SM::B_ATOM);
            if (rank == 0) {
              mbar_arrive_expect_tx(&full[s], ATOM_TX);
              mbar_arrive_expect_tx(&full_hi[s], ATOM_TX);
            }
#pragma unroll
            for (int j = 0; j < SM::KA; ++j) {
              // atoms past K read as zeros (TMA out-of-bounds fill) and add nothing
              const uint32_t lead_full = mapa_shared(smem_addr(j == 0 ? &full[s] : &full_hi[s]), lead);
              const int k0 = (kb * SM::KA + j) * GEMM_BK;
              tma_load_2d_pair(st + j * SM::A_ATOM, &tmA, lead_full, k0, arow, pol_a);
              tma_load_2d_pair(st + SM::A_BYTES + j * SM::B_ATOM, &tmB, lead_full, k0, brow, pol_b);
            }
          }
        }
      }
      if (W4) {
        // drain: no copy may still be landing in shared memory when the CTA exits
        const uint32_t n_issued = it;
        const uint32_t first = n_issued > static_cast<uint32_t>(S) ? n_issued - S : 0u;
        for (uint32_t j = first; j < n_issued; ++j) {
          int dummy = 0;
          mbar_wait(&full[j % S], (j / S) & 1u, &dummy, SITE_DRAIN);
        }
      }
      // int8: the leader's MMA thread consumed every stage, so both CTAs' copies
      // have landed before it passes the final pair barrier
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && rank == 0) {
      uint32_t it = 0, local = 0;
      bool ok = true;
      while (ok && next_seg(seg)) {
        const uint32_t b = local & 1u;
        const uint32_t use = local >> 1;
        if (!mbar_wait(&tmem_empty[b], (use & 1u) ^ 1u, abort_flag, SITE_MMA_TMEM)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + b * BN;
        for (int kb = seg.kb0; kb < seg.kb1; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(W4 ? &conv[s] : &full[s], ph, abort_flag, SITE_MMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(smem + s * SM::STAGE);
          const uint32_t sb = sa + SM::A_BYTES;
#pragma unroll
          for (int j = 0; j < SM::KA; ++j) {
            if (!W4 && j == 1) {
              if (!mbar_wait(&full_hi[s], ph, abort_flag, SITE_MMA_FULL)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
#pragma unroll
            for (int k = 0; k < GEMM_BK / GEMM_UMMA_K; ++k) {
              mma_s8_pair(d, sw128_kmajor_desc(sa + j * SM::A_ATOM + k * GEMM_UMMA_K),
                          sw128_kmajor_desc(sb + j * SM::B_ATOM + k * GEMM_UMMA_K), IDESC,
                          (kb > seg.kb0 || j > 0 || k > 0) ? 1u : 0u);
            }
          }
          if (!ok) break;
          mma_commit_pair_mc(&empty[s], pair_mask);
        }
        if (!ok) break;
        mma_commit_pair_mc(&tmem_full[b], pair_mask);
        ++local;
      }
      // every MMA this thread issued must be complete before TMEM is released
      mma_commit_pair(drain);
      int never = 0;
      mbar_wait(drain, 0u, &never, SITE_DRAIN);
    }
  } else if (warp < 2 + PAIR_EPI_WARPS) {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;          // 0..7
    const int q = warp & 3;           // TMEM lane quadrant this warp may access
    const int h = ew >> 2;            // column half of the tile: 128 columns each
    uint32_t local = 0;
    uint32_t sync_phase = 0;
    auto epi_rendezvous = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_sync);
      const bool r = mbar_wait(epi_sync, sync_phase & 1u, abort_flag, SITE_EPI_SYNC);
      ++sync_phase;
      __syncwarp();
      return r;
    };
    constexpr int OC = (EPI == EPI_BF16) ? 64 : 32;  // output columns per 128-byte staged row
    uint8_t* buf = smem + SM::staging_offset(S) + ew * 4096;
    // columns of a tile this warp finalises: its 128-column half, or in SPLIT
    // mode 64 columns of its own pair's half of the tile
    constexpr int FC = SPLIT ? 64 : 128;
    // A finalised tile's accumulator buffer goes back to the MMA when the next
    // tile begins: after the last tile nothing waits for it, and its
    // cluster-scope arrive would only delay the CTA's exit.
    int pending = -1;
    while (next_seg(seg)) {
      if (pending >= 0) {
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_addr(&tmem_empty[pending]), lead));
        pending = -1;
      }
      const uint32_t b = local & 1u;
      const uint32_t use = local >> 1;
      int ta, tb;
      tile_coords(a, seg.tile, ta, tb);
      const int m0 = ta * 256 + static_cast<int>(rank) * 128 + 32 * q;  // first row of this warp
      const int fcol = SPLIT ? static_cast<int>(pq) * 128 + h * 64 : h * 128;
      const int ncol0 = tb * BN + fcol;  // first output column this warp finalises
      // output scales, loaded while the accumulators are still being computed:
      // lane l holds s_row of column ncol0 + 32 c + l
      const int m = m0 + lane;
      float st = 0.f;
      float srl[FC / 32];
#pragma unroll
      for (int c = 0; c < FC / 32; ++c) srl[c] = 0.f;
      if (EPI != EPI_S32) {
        if (m < a.M) st = __ldg(a.s_tok + m) * (W4 ? 0.0625f : 1.0f);
#pragma unroll
        for (int c = 0; c < FC / 32; ++c) {
          const int n = ncol0 + 32 * c + lane;
          if (n < a.N) srl[c] = __ldg(a.s_row + n);
        }
      }
      const bool got = mbar_wait(&tmem_full[b], use & 1u, abort_flag, SITE_EPI_FULL);
      __syncwarp();
      if (!got) break;
      tc_fence_after();
      const uint32_t tq = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + b * BN;
      const uint32_t tbase = tq + h * 128;  // this warp's 128-column half (stream-K path)
      const uint32_t lead_tmem_empty = mapa_shared(smem_addr(&tmem_empty[b]), lead);

      // SPLIT: the CTA of the other pair with the same rows finalises the
      // columns this warp sends, and sends the ones this warp finalises.  The
      // receive area (the first 64 KB of the stage ring) holds, per warp, its
      // 32 rows x 64 columns as 2 chunks of 32 columns, each 8 x (32 lanes x
      // 16 bytes).
      const uint32_t recv_off = static_cast<uint32_t>(q * 2 + h) * 8192u;
      if (SPLIT) {
        const uint32_t other = pq ? crank - 2u : crank + 2u;
        if (ew == 0 && lane == 0) {
          // this CTA's MMAs are complete, so its stage ring is free: tell the
          // other CTA with a 16-byte async copy into its signal slot, which
          // completes bytes on its `ready` barrier (a cluster-scope release
          // arrive would take ~0.8 us); this CTA's own `ready` completes when
          // the other CTA's copy lands
          mbar_arrive_expect_tx(recv, SPLIT_RECV_BYTES);
          mbar_arrive_expect_tx(ready, 16u);
          bulk_copy_to_cluster(mapa_shared(smem_addr(sig + 16), other), sig, 16u,
                               mapa_shared(smem_addr(ready), other));
        }
        // stage the columns the other CTA finalises in this CTA's own ring (above
        // the receive area), in the receive layout, then copy the warp's 8 KB in
        // one bulk copy once the other CTA's ring is free
        const int scol = (1 - static_cast<int>(pq)) * 128 + h * 64;
        uint8_t* sendbuf = smem + SPLIT_RECV_BYTES + recv_off;
#pragma unroll 1
        for (int cl = 0; cl < 2; ++cl) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tq + scol + cl * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4)
            st_shared_v4(sendbuf + (cl * 8 + j4) * 512 + lane * 16, r[4 * j4], r[4 * j4 + 1],
                         r[4 * j4 + 2], r[4 * j4 + 3]);
        }
        fence_proxy_async_smem();
        const bool go = mbar_wait(ready, 0u, abort_flag, SITE_SPLIT);
        __syncwarp();
        if (!go) break;
        if (lane == 0)
          bulk_copy_to_cluster(mapa_shared(smem_addr(smem), other) + recv_off, sendbuf, 8192u,
                               mapa_shared(smem_addr(recv), other));
        const bool got_partial = mbar_wait(recv, 0u, abort_flag, SITE_SPLIT);
        __syncwarp();
        if (!got_partial) break;
      }

      // A split tile: every contributing pair adds its int32 partial into one
      // accumulator per CTA of the tile (bulk reductions performed at L2); the
      // pair that completes the tile's count reads it back, re-zeroes it and
      // writes the output.
      const int u_sk = seg.tile - a.dp_tiles;
      int32_t* acc_tile = a.ws_acc + static_cast<size_t>(2 * u_sk + rank) * (GEMM_BM * BN);
      if (seg.partial) {
#pragma unroll 1
        for (int cl = 0; cl < 4; ++cl) {  // this warp's 32-column chunks
          const int c = h * 4 + cl;
          uint32_t r[32];
          tmem_ld_32x32b_x32(tbase + cl * 32, r);
          tmem_ld_wait();
          if (lane == 0) bulk_wait_group_read<0>();  // the previous reduction has read buf
          __syncwarp();
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4)
            st_shared_v4(buf + (j4 * 32 + lane) * 16, r[4 * j4], r[4 * j4 + 1], r[4 * j4 + 2],
                         r[4 * j4 + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            bulk_reduce_add_s32(acc_tile + (c * 4 + q) * 1024, buf, 4096);
            bulk_commit_group();
          }
        }
      }
      bool finalize = !seg.partial;
      if (seg.partial) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(lead_tmem_empty);
        if (lane == 0) {
          bulk_wait_group<0>();  // this warp's reductions are performed
          fence_proxy_async_global();
        }
        // the rendezvous orders every warp's performed reductions before the
        // counting thread's release below (one gpu-scope ordering point, not a
        // fence in every thread)
        __syncwarp();
        if (!epi_rendezvous()) break;
        if (ew == 0 && lane == 0) {
          const int c_lo = sk_owner(a, u_sk * a.num_kb);
          const int c_hi = sk_owner(a, (u_sk + 1) * a.num_kb - 1);
          const unsigned prev = atomic_add_acq_rel_gpu(&a.ws_counts[2 * u_sk + rank], 1u);
          const bool last = prev + 1u == static_cast<unsigned>(c_hi - c_lo + 1);
          if (last) a.ws_counts[2 * u_sk + rank] = 0u;
          *last_flag = last ? 1 : 0;
        }
        if (!epi_rendezvous()) break;
        // the counting thread acquired the other units' sums; the rendezvous
        // carries that to every thread of the CTA
        finalize = *last_flag != 0;
      }
      if (finalize && EPI == EPI_SWIGLU) {
        // MLP boundary: the warp's 128 accumulator columns are four blocks of
        // 16 gate and 16 up columns; their 64 outputs fill one staged 128-byte
        // row per token, stored with one TMA store at column ncol0 / 2
        if (lane == 0) bulk_wait_group_read<0>();  // the previous store has read buf
        __syncwarp();
        const int sw = lane & 7;
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // unrolled: srl[c] stays in registers
          uint32_t r[32];
          if (!seg.partial) {
            tmem_ld_32x32b_x32(tq + fcol + 32 * c, r);
            tmem_ld_wait();
          } else {
            // the tile's sum; leave the accumulator at zero for the next call
            uint4* base = reinterpret_cast<uint4*>(acc_tile) + ((h * 4 + c) * 4 + q) * 8 * 32 + lane;
            uint4 v[8];
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) v[j4] = __ldcg(base + j4 * 32);
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              __stcg(base + j4 * 32, z);
              r[4 * j4] = v[j4].x;
              r[4 * j4 + 1] = v[j4].y;
              r[4 * j4 + 2] = v[j4].z;
              r[4 * j4 + 3] = v[j4].w;
            }
          }
          float sr[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) sr[j] = __shfl_sync(0xffffffffu, srl[c], j);
          uint32_t w[8];
          swiglu16(r, st, sr, w);
          st_shared_v4(buf + lane * 128 + (((2 * c) ^ sw) << 4), w[0], w[1], w[2], w[3]);
          st_shared_v4(buf + lane * 128 + (((2 * c + 1) ^ sw) << 4), w[4], w[5], w[6], w[7]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmY, buf, ncol0 / 2, m0);
          bulk_commit_group();
        }
      } else if (finalize) {
#pragma unroll
        for (int oc = 0; oc < FC / OC; ++oc) {
          uint32_t r0[32], r1[32];
          if (!seg.partial) {
            tmem_ld_32x32b_x32(tq + fcol + oc * OC, r0);
            if (OC == 64) tmem_ld_32x32b_x32(tq + fcol + oc * OC + 32, r1);
            tmem_ld_wait();
            if (SPLIT) {
              // add the other pair's half-K partial (exact int32 sums)
              const uint8_t* rb = smem + recv_off;
              const int c0 = oc * (OC / 32);
#pragma unroll
              for (int j4 = 0; j4 < 8; ++j4) {
                const uint4 p0 = ld_shared_v4(rb + (c0 * 8 + j4) * 512 + lane * 16);
                r0[4 * j4] += p0.x;
                r0[4 * j4 + 1] += p0.y;
                r0[4 * j4 + 2] += p0.z;
                r0[4 * j4 + 3] += p0.w;
                if (OC == 64) {
                  const uint4 p1 = ld_shared_v4(rb + ((c0 + 1) * 8 + j4) * 512 + lane * 16);
                  r1[4 * j4] += p1.x;
                  r1[4 * j4 + 1] += p1.y;
                  r1[4 * j4 + 2] += p1.z;
                  r1[4 * j4 + 3] += p1.w;
                }
              }
            }
          } else {
            // the tile's sum; leave the accumulator at zero for the next call
            const int c0 = h * 4 + oc * (OC / 32);
            uint4* base = reinterpret_cast<uint4*>(acc_tile);
            uint4 v0[8], v1[8];
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              v0[j4] = __ldcg(base + ((c0 * 4 + q) * 8 + j4) * 32 + lane);
              if (OC == 64) v1[j4] = __ldcg(base + (((c0 + 1) * 4 + q) * 8 + j4) * 32 + lane);
            }
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              __stcg(base + ((c0 * 4 + q) * 8 + j4) * 32 + lane, z);
              if (OC == 64) __stcg(base + (((c0 + 1) * 4 + q) * 8 + j4) * 32 + lane, z);
              r0[4 * j4] = v0[j4].x;
              r0[4 * j4 + 1] = v0[j4].y;
              r0[4 * j4 + 2] = v0[j4].z;
              r0[4 * j4 + 3] = v0[j4].w;
              if (OC == 64) {
                r1[4 * j4] = v1[j4].x;
                r1[4 * j4 + 1] = v1[j4].y;
                r1[4 * j4 + 2] = v1[j4].z;
                r1[4 * j4 + 3] = v1[j4].w;
              }
            }
          }
          if (lane == 0) bulk_wait_group_read<0>();  // the previous store has read buf
          __syncwarp();
          const int sw = lane & 7;
          if (EPI == EPI_BF16) {
#pragma unroll
            for (int c16 = 0; c16 < 8; ++c16) {
              const uint32_t* rr = c16 < 4 ? r0 : r1;
              const int jb = (c16 & 3) * 8;
              // s_row of columns oc * 64 + c16 * 8 + 0..7, held by lanes jb..jb+7
              const float srv = srl[oc * 2 + (c16 >> 2)];
              float sr[8];
#pragma unroll
              for (int hh = 0; hh < 8; ++hh) sr[hh] = __shfl_sync(0xffffffffu, srv, jb + hh);
              uint32_t w[4];
#pragma unroll
              for (int hh = 0; hh < 4; ++hh) {
                const float y0 = static_cast<float>(static_cast<int32_t>(rr[jb + 2 * hh])) * st * sr[2 * hh];
                const float y1 = static_cast<float>(static_cast<int32_t>(rr[jb + 2 * hh + 1])) * st * sr[2 * hh + 1];
                w[hh] = pack_bf16x2(y0, y1);
              }
              st_shared_v4(buf + lane * 128 + ((c16 ^ sw) << 4), w[0], w[1], w[2], w[3]);
            }
          } else {
            const int sh = W4 ? 4 : 0;
#pragma unroll
            for (int c16 = 0; c16 < 8; ++c16) {
              st_shared_v4(buf + lane * 128 + ((c16 ^ sw) << 4),
                           static_cast<uint32_t>(static_cast<int32_t>(r0[4 * c16]) >> sh),
                           static_cast<uint32_t>(static_cast<int32_t>(r0[4 * c16 + 1]) >> sh),
                           static_cast<uint32_t>(static_cast<int32_t>(r0[4 * c16 + 2]) >> sh),
                           static_cast<uint32_t>(static_cast<int32_t>(r0[4 * c16 + 3]) >> sh));
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmY, buf, ncol0 + oc * OC, m0);
            bulk_commit_group();
          }
        }
      }
      if (!seg.partial) {
        tc_fence_before();
        __syncwarp();
        pending = static_cast<int>(b);
      }
      ++local;
    }
    // the staged outputs must have been read before the CTA exits; the global
    // writes themselves complete before the grid does
    if (lane == 0) bulk_wait_group_read<0>();
  } else if (W4) {
    // ------------------------------------------------------------ int4 unpack
    // Each thread reads its share of every packed atom of the stage (4 x 16
    // bytes per atom), the four warps meet (bounded), then each writes the
    // unpacked 128-byte swizzled rows, which overwrite the packed bytes.
    const int ct = threadIdx.x - 32 * (2 + PAIR_EPI_WARPS);  // 0..127
    uint32_t it = 0, cv_phase = 0;
    bool ok = true;
    while (ok && next_seg(seg)) {
      for (int kb = seg.kb0; kb < seg.kb1; ++kb, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1u;
        if (!mbar_wait(&full[s], ph, abort_flag, SITE_CONV_FULL)) {
          ok = false;
          break;
        }
        uint8_t* st = smem + s * SM::STAGE;
        uint4 pk[SM::KA][4];
#pragma unroll
        for (int j = 0; j < SM::KA; ++j) {
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int idx = ct + 128 * t, r = idx >> 2, pc = idx & 3;
            pk[j][t] = ld_shared_v4(st + SM::A_BYTES + j * SM::B_ATOM + SM::PACKED_OFF + r * 64 +
                                    pc * 16);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(cv_sync);
        const bool met = mbar_wait(cv_sync, cv_phase & 1u, abort_flag, SITE_CONV_FULL);
        ++cv_phase;
        __syncwarp();
        if (!met) {
          ok = false;
          break;
        }
#pragma unroll
        for (int j = 0; j < SM::KA; ++j) {
          uint8_t* unp = st + SM::A_BYTES + j * SM::B_ATOM;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int idx = ct + 128 * t, r = idx >> 2, pc = idx & 3;
            const uint32_t w[4] = {pk[j][t].x, pk[j][t].y, pk[j][t].z, pk[j][t].w};
            uint32_t o[8];
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
              const uint32_t lo = (w[hh] << 4) & 0xF0F0F0F0u;
              const uint32_t hi = w[hh] & 0xF0F0F0F0u;
              o[2 * hh] = __byte_perm(lo, hi, 0x5140);
              o[2 * hh + 1] = __byte_perm(lo, hi, 0x7362);
            }
            const int sw = r & 7;
            st_shared_v4(unp + r * 128 + (((2 * pc) ^ sw) << 4), o[0], o[1], o[2], o[3]);
            st_shared_v4(unp + r * 128 + (((2 * pc + 1) ^ sw) << 4), o[4], o[5], o[6], o[7]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int cw = ct >> 5;  // converter warp 0..3
          if (rank == 0) {
            // leader: a local arrive; warp 0's also expects the partner's signals
            if (cw == 0)
              mbar_arrive_expect_tx(&conv[s], 4u * 16u);
            else
              mbar_arrive(&conv[s]);
          } else {
            // partner: its expanded rows are visible to the async proxy (fence
            // above); a 16-byte async copy into the leader's slot completes
            // bytes on the leader's barrier
            bulk_copy_to_cluster(mapa_shared(smem_addr(sig + cw * 16), lead), sig + cw * 16, 16u,
                                 mapa_shared(smem_addr(&conv[s]), lead));
          }
        }
      }
    }
  }

  __syncwarp();  // roles ran on single lanes: reconverge before the aligned barrier
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no cross-CTA arrive, copy or MMA can still target either CTA
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, SM::TMEM_COLS);
  }
}

}  // namespace convrot
