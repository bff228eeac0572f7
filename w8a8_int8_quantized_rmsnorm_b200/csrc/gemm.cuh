// W8A8 / W4A8 ConvRot linear on the 5th-generation tensor core.
//
//   acc[m, n] = sum_k Xq[m, k] * Wq[n, k]                 (exact int32)
//   Y[m, n]   = bf16_rn(float(acc) * s_tok[m] * s_row[n])
//
// ("MOSS-Image Qwen3.5-9B text encoder, INT8 (W8A8, ConvRot)", file table,
// "Matmul" row; the int4 weight layout of "MossInt4", "Format".)
//
// Kernel structure (one CTA per SM, persistent):
//   warp 0      TMA producer: int8 tiles of both operands, one or two 128-byte
//               K atoms per stage, 128-byte swizzle, into a ring of
//               shared-memory stages;
//   warp 1      allocates TMEM and issues tcgen05.mma kind::i8 (one thread),
//               128 x BN x 32 per instruction, s32 accumulators in TMEM,
//               two accumulator buffers so the epilogue of one tile overlaps
//               the main loop of the next;
//   warps 2-5   epilogue: tcgen05.ld of the accumulators, dequantisation to
//               bf16 (or raw int32), staged in shared memory in the output's
//               layout and written with TMA stores;
//   warps 6-9   (int4 weights only) unpack two signed nibbles per byte into
//               the swizzled int8 stage the MMA reads.  A nibble n is written
//               as the byte n * 16 (the nibble in the high half), so the MMA
//               accumulates 16 * acc exactly and the epilogue divides by 16.
//
// Operand roles.  Operand A fills the MMA's M = 128 rows, operand B its N = BN
// columns.  For M > 128 tokens A = activations and B = weights (BN = 256).
// For M <= 128 the roles swap (A = weights, B = tokens, BN = 16..128), so the
// 128-row tensor-core dimension is filled by weight rows and every weight
// byte is streamed exactly once.
//
// Work split.  Output tiles are ordered in groups of 8 A-tiles for L2 reuse.
// Whole waves of tiles are handed out round-robin (data-parallel).  The last
// one to two waves are split evenly by pipeline stage over all CTAs
// (stream-K).  A CTA whose range covers only part of a tile adds its int32
// partial tile into the tile's accumulator in the workspace (bulk add
// reductions performed at L2), then increments the tile's counter; the CTA
// that brings the counter to the number of contributors reads the sum back,
// re-zeroes the accumulator and the counter, and writes the output.  Integer
// addition makes the result independent of arrival order.  No CTA ever waits
// on another CTA.
#pragma once

#include "ptx.cuh"

namespace convrot {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 128;  // int8 elements (bytes) of K per swizzle atom
constexpr int GEMM_UMMA_K = 32;
constexpr int GEMM_MAX_STAGES = 16;
constexpr int GEMM_GROUP_A = 8;  // rasterisation group of the single-CTA kernels
// decode kernels: before the dependency wait, the weights of this many K atoms
// beyond the ring's first fill go towards L2
constexpr int GEMM_PREFETCH_ATOMS = 8;
// 128-byte K atoms per pipeline stage.  A single thread issues every
// tcgen05.mma, and each MMA issue, stage wait and commit costs that thread tens
// of cycles: with one atom (four 32-deep MMAs) per stage the issuing thread
// needs more than the 512 tensor-pipe cycles of a 128 x 256 x 128 (or pair
// 256 x 256 x 128) step and the pipe idles between steps.  Two atoms per stage
// halve the waits and commits per MMA.  Int4 weights on the single-CTA
// kernel keep one atom (its stage also holds the packed tile); the pair
// kernel unpacks them in place and takes two.
__host__ __device__ constexpr int gemm_katoms(bool w4, bool pair, bool swap) {
  return w4 ? (pair ? 2 : 1) : ((pair || swap) ? 2 : 1);
}

// K atoms (64 elements each) per stage of the weight-only path.  Its weights
// are expanded into tensor memory, so a stage holds only the landed int8
// weights and the tokens: four atoms (32 KB of weights, the int8 decode
// stage's share) for token tiles up to 64, two for 128 (where four would
// leave two stages).  Halving the stages per weight byte took M = 16 from
// 37.6 to 30.7 us (measured).
__host__ __device__ constexpr int wbf_katoms(int bn) { return bn <= 64 ? 4 : 2; }
constexpr int EPI_BF16 = 0;
constexpr int EPI_S32 = 1;
// SiLU(gate) * up of the MLP boundary: the weight rows alternate in blocks of
// SWIGLU_BLOCK gate rows and SWIGLU_BLOCK up rows, and the output has half as
// many columns as the weight has rows
constexpr int EPI_SWIGLU = 2;
constexpr int SWIGLU_BLOCK = 16;

struct GemmArgs {
  int M, N, K;
  int rowsA, rowsB;  // rows of operands A and B
  int tilesA, tilesB;
  int group_a;       // tiles run in groups of this many A tiles, all B tiles of a group first
  int num_tiles;
  int num_kb;        // pipeline stages of K per tile (KA atoms of 128 bytes each)
  int stages;
  int dp_tiles;      // tiles [0, dp_tiles) are data-parallel
  int sk_iters;      // (num_tiles - dp_tiles) * num_kb
  int sk_q, sk_r;    // stream-K split: first sk_r CTAs get sk_q + 1 iterations
  const float* s_tok;
  const float* s_row;
  int srow_vec;  // s_row is 16-byte aligned: vector loads in the epilogue
  void* out;
  int32_t* ws_acc;       // [split tiles][CTAs per unit][BM * BN] int32 accumulators
  unsigned* ws_counts;   // [split tiles][CTAs per unit] arrival counters
};

struct Segment {
  int tile, kb0, kb1;
  bool partial;
  int slot;
};

struct Schedule {
  const GemmArgs* p;
  int cta, ncta;
  int dp_next;
  int sk_begin, sk_end, sk_cur;

  // unit = CTA (or CTA pair) index, nunits = number of units in the grid
  __device__ void init(const GemmArgs& a, int unit, int nunits) {
    p = &a;
    cta = unit;
    ncta = nunits;
    dp_next = cta;
    sk_begin = cta * a.sk_q + min(cta, a.sk_r);
    sk_end = sk_begin + a.sk_q + (cta < a.sk_r ? 1 : 0);
    sk_cur = sk_begin;
  }
  __device__ bool next(Segment& s) {
    if (dp_next < p->dp_tiles) {
      s.tile = dp_next;
      s.kb0 = 0;
      s.kb1 = p->num_kb;
      s.partial = false;
      s.slot = -1;
      dp_next += ncta;
      return true;
    }
    if (sk_cur < sk_end) {
      const int u = sk_cur / p->num_kb;
      s.kb0 = sk_cur - u * p->num_kb;
      s.kb1 = min(p->num_kb, s.kb0 + (sk_end - sk_cur));
      s.tile = p->dp_tiles + u;
      s.partial = !(s.kb0 == 0 && s.kb1 == p->num_kb);
      s.slot = 2 * cta + (sk_cur == sk_begin ? 0 : 1);
      sk_cur += s.kb1 - s.kb0;
      return true;
    }
    return false;
  }
};

// CTA that owns stream-K iteration i.
__device__ __forceinline__ int sk_owner(const GemmArgs& a, int i) {
  const int big = a.sk_r * (a.sk_q + 1);
  if (i < big) return i / (a.sk_q + 1);
  return a.sk_r + (i - big) / a.sk_q;
}
__device__ __forceinline__ int sk_begin_of(const GemmArgs& a, int c) {
  return c * a.sk_q + min(c, a.sk_r);
}

__device__ __forceinline__ void tile_coords(const GemmArgs& a, int tile, int& ta, int& tb) {
  const int per_group = a.group_a * a.tilesB;
  const int group = tile / per_group;
  const int first = group * a.group_a;
  const int ga = min(a.group_a, a.tilesA - first);
  const int local = tile - group * per_group;
  ta = first + local % ga;
  tb = local / ga;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// SiLU(g) * u in fp32: g / (1 + e^-g) * u.  For g far below zero e^-g is
// infinite and the quotient is a signed zero, the function's limit.
__device__ __forceinline__ float silu_mul(float g, float u) {
  return g / (1.0f + __expf(-g)) * u;
}

// Sixteen outputs of the MLP boundary from one 32-column accumulator chunk
// whose first 16 columns are gate rows and last 16 the matching up rows:
// h_j = SiLU(acc_j * st * sr_j) * (acc_{16+j} * st * sr_{16+j}), as 8 bf16x2.
__device__ __forceinline__ void swiglu16(const uint32_t (&r)[32], float st, const float (&sr)[32],
                                         uint32_t (&w)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float g0 = static_cast<float>(static_cast<int32_t>(r[2 * j])) * st * sr[2 * j];
    const float g1 = static_cast<float>(static_cast<int32_t>(r[2 * j + 1])) * st * sr[2 * j + 1];
    const float u0 = static_cast<float>(static_cast<int32_t>(r[16 + 2 * j])) * st * sr[16 + 2 * j];
    const float u1 = static_cast<float>(static_cast<int32_t>(r[17 + 2 * j])) * st * sr[17 + 2 * j];
    w[j] = pack_bf16x2(silu_mul(g0, u0), silu_mul(g1, u1));
  }
}

// Shared-memory plan (offsets from a 1024-byte aligned base).  W4 here means
// "a converter stage" (int4 or the weight-only path); KAO overrides the K atoms
// per stage.  A converter stage's packed weight atom (64 bytes per row) lands
// in the upper half of its weight atom's slot and is expanded in place to the
// 128-byte swizzled rows the MMA reads, so a stage holds no separate packed
// area.  TSA (weight-only path, swapped roles): the stage's weights are only
// the landed int8 tile (boxes of two 64-element atoms = 128 bytes per row,
// 128-byte swizzle); their bf16 expansion is the MMA's A operand in tensor
// memory, up to TSA_BUFS stages' worth of columns after the two accumulator
// buffers.
template <int BN, bool W4, bool SWAP, int KAO = 0, bool TSA = false>
struct GemmSmem {
  static constexpr int KA = KAO ? KAO : gemm_katoms(W4, false, SWAP);
  // one K atom of the A tile: 128 bytes per row, or the landed 64 of TSA
  static constexpr int A_ATOM = TSA ? GEMM_BM * (GEMM_BK / 2) : GEMM_BM * GEMM_BK;
  static constexpr int B_ATOM = BN * GEMM_BK;
  static constexpr int A_BYTES = KA * A_ATOM;
  static constexpr int B_BYTES = KA * B_ATOM;
  static constexpr int W_ROWS = SWAP ? GEMM_BM : BN;                // rows of the weight tile
  static constexpr int P_ATOM = W4 ? W_ROWS * (GEMM_BK / 2) : 0;  // packed int4 / int8 weight atom
  static constexpr int P_BYTES = KA * P_ATOM;                      // packed bytes per stage
  static constexpr int PACKED_OFF = TSA ? 0 : W_ROWS * (GEMM_BK / 2);  // inside a weight atom's slot
  static constexpr int STAGE = A_BYTES + B_BYTES;
  // per epilogue warp two 4 KB staging buffers (32 rows x 128 B) for output
  // stores and split-tile reductions
  static constexpr int STAGING = 4 * 2 * 4096;
  static constexpr int ACC_STRIDE = BN < 32 ? 32 : BN;  // TMEM columns per accumulator buffer
  // TSA: A buffers of one stage each (64 bf16 = 32 columns per K atom), at
  // most TSA_BUFS of them and fewer than the stages (the converter reuses a
  // buffer once its stage's slot has been released, which must not have
  // happened twice since)
  static constexpr int TSA_BUFS = 4;
  static constexpr int TSA_COLS = KA * (GEMM_BK / 4);
  static constexpr int TSA_COL0 = 2 * ACC_STRIDE;
  static constexpr int TMEM_COLS = TSA ? 512 : 2 * ACC_STRIDE;
  static constexpr int TSA_MAXBUF = (512 - TSA_COL0) / TSA_COLS;  // what tensor memory holds
  static_assert(!TSA || TSA_MAXBUF >= 1, "tensor memory holds 512 columns");
  static_assert(!TSA || KA % 2 == 0, "a TSA stage lands 128-byte weight rows: two bf16 atoms");
  static constexpr int CW = BN < 32 ? BN : 32;  // accumulator columns per tcgen05.ld
  __host__ __device__ static int staging_offset(int stages) { return stages * STAGE; }
  __host__ __device__ static int bar_offset(int stages) { return stages * STAGE + STAGING; }
  // full, empty, conv: stages each; tmem_full, tmem_empty: 2 each; drain,
  // epi_sync, cv_sync; + scalars
  __host__ __device__ static int total(int stages) {
    return bar_offset(stages) + (3 * GEMM_MAX_STAGES + 7) * 8 + 64;
  }
};

// Four int8 codes q (one 32-bit word, lowest byte first) -> four bf16,
// exactly, on the full-rate ALU: u = q + 128 (the sign bit flipped) goes into
// the low byte of the fp32 2^23 + u, and subtracting 2^23 + 128 leaves q; q
// has at most 8 significant bits, so its bf16 is the upper half.  lo holds
// codes 0, 1 and hi codes 2, 3, the lower code in the low half of each.
__device__ __forceinline__ void i8x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const uint64_t m01 = static_cast<uint64_t>(__byte_perm(u, 0x4B000000u, 0x7540)) |
                       (static_cast<uint64_t>(__byte_perm(u, 0x4B000000u, 0x7541)) << 32);
  const uint64_t m23 = static_cast<uint64_t>(__byte_perm(u, 0x4B000000u, 0x7542)) |
                       (static_cast<uint64_t>(__byte_perm(u, 0x4B000000u, 0x7543)) << 32);
  const uint64_t bias = 0x4B0000804B000080ull;  // (2^23 + 128, 2^23 + 128)
  uint64_t f01, f23;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(f01) : "l"(m01), "l"(bias));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(f23) : "l"(m23), "l"(bias));
  lo = __byte_perm(static_cast<uint32_t>(f01), static_cast<uint32_t>(f01 >> 32), 0x7632);
  hi = __byte_perm(static_cast<uint32_t>(f23), static_cast<uint32_t>(f23 >> 32), 0x7632);
}

// Accumulator value: int32 for the integer MMAs, fp32 bits for kind::f16.
template <bool F32ACC>
__device__ __forceinline__ float acc_value(uint32_t r) {
  return F32ACC ? __uint_as_float(r) : static_cast<float>(static_cast<int32_t>(r));
}

// One CTA per SM.  Registers are allocated per SM sub-partition (16K each, a
// CTA's warps spread over four): with 6 (10) warps, two (three) share one, so
// 255 (168) registers per thread is the most a launch can use.
//
// WBF (weight-only path, always the swapped roles): the activation operand is
// bf16 (already rotated), the MMA is kind::f16 with an fp32 accumulator and
// the epilogue scales by s_row only.  The converter warps expand the int8
// weight tile to bf16 into tensor memory as the MMA's A operand (TSA), each
// converter thread taking one weight row of its warp's lane quadrant, so a
// stage's slot holds only the landed int8 weights and the tokens.  (Expanding
// into shared memory, as the int4 path does, measured 2x slower at M = 512,
// N = K = 4096 and 5 % slower at M = 2048, N = 24576.)
template <int BN, bool SWAP, bool W4, int EPI, bool WBF = false>
__global__ void __launch_bounds__((W4 || WBF) ? 320 : 192) __maxnreg__((W4 || WBF) ? 168 : 255)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmY, GemmArgs a) {
  constexpr bool CONV = W4 || WBF;  // a converter stage between TMA and the MMA
  static_assert(!(W4 && WBF), "int4 weights have no weight-only path");
  static_assert(!(WBF && EPI == EPI_SWIGLU), "the weight-only path has no SwiGLU epilogue");
  static_assert(!WBF || SWAP, "the weight-only path runs the swapped roles");
  constexpr bool TSA = WBF;  // expanded weights in tensor memory
  using SM = GemmSmem<BN, CONV, SWAP, WBF ? wbf_katoms(BN) : 0, TSA>;
  static_assert(!W4 || SM::KA == 1, "int4 stages hold one K atom");
  constexpr int CW = SM::CW;
  pdl_launch_dependents();  // the grid is co-resident: dependents only take idle SMs
  constexpr uint32_t IDESC = WBF ? idesc_bf16_f32(GEMM_BM, BN) : idesc_s8s8s32(GEMM_BM, BN);

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int S = a.stages;
  // TSA: tensor-memory A buffers in use, fewer than the stages
  const int nbufs = TSA ? min(min(SM::TSA_BUFS, S - 1), SM::TSA_MAXBUF) : 1;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::bar_offset(S));
  uint64_t* empty = full + GEMM_MAX_STAGES;
  uint64_t* conv = empty + GEMM_MAX_STAGES;
  uint64_t* tmem_full = conv + GEMM_MAX_STAGES;
  uint64_t* tmem_empty = tmem_full + 2;
  uint64_t* drain = tmem_empty + 2;
  uint64_t* epi_sync = drain + 1;  // rendezvous of the four epilogue warps
  uint64_t* cv_sync = epi_sync + 1;  // rendezvous of the four converter warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cv_sync + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&conv[s], 4);  // the four converter warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tmem_full[b], 1);
      mbar_init(&tmem_empty[b], 4);
    }
    mbar_init(drain, 1);
    mbar_init(epi_sync, 4);
    mbar_init(cv_sync, 4);
    *abort_flag = 0;
    *last_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, SM::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (SWAP && threadIdx.x == 64) {
    // Decode shapes: the previous kernel (the rotate-quantise of a few
    // tokens) occupies few SMs, so this CTA may wait here for a while.  The
    // weights never come from that kernel: start this CTA's first stages of
    // them towards L2 meanwhile.  A prefetch is only a hint (L2 is coherent),
    // so it is safe before griddepcontrol.wait.  (Lane 0 of the first
    // epilogue warp, idle until the first accumulators are ready.)
    Schedule first;
    first.init(a, blockIdx.x, gridDim.x);
    Segment s0;
    if (first.next(s0)) {
      int ta, tb;
      tile_coords(a, s0.tile, ta, tb);
      const int kend = min(s0.kb1, s0.kb0 + S + GEMM_PREFETCH_ATOMS / SM::KA);
      for (int kb = s0.kb0; kb < kend; ++kb) {
        if (TSA) {  // 128-byte boxes per weight row
          for (int h = 0; h < SM::KA / 2; ++h)
            tma_prefetch_l2_2d(&tmA, (kb * SM::KA / 2 + h) * GEMM_BK, ta * GEMM_BM);
        } else {
          for (int j = 0; j < SM::KA; ++j) {
            const int atom = kb * SM::KA + j;
            tma_prefetch_l2_2d(&tmA, (W4 || WBF) ? atom * (GEMM_BK / 2) : atom * GEMM_BK,
                               ta * GEMM_BM);
          }
        }
      }
    }
  }
  pdl_wait();  // operands, scales and the output may belong to the previous kernel

  Schedule sched;
  sched.init(a, blockIdx.x, gridDim.x);
  Segment seg;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_a = SWAP ? policy_evict_first() : policy_evict_last();
      const uint64_t pol_b = SWAP ? policy_evict_last() : policy_evict_first();
      uint32_t tx = 0;
      if (CONV) {
        tx = SWAP ? (SM::P_BYTES + SM::B_BYTES) : (SM::A_BYTES + SM::P_BYTES);
      } else {
        tx = SM::A_BYTES + SM::B_BYTES;
      }
      uint32_t it = 0;
      bool ok = true;
      constexpr int KA = SM::KA;
      // innermost TMA coordinate of K atom `atom`: int8 bytes, or half of that
      // for packed int4 weights; WBF atoms are 64 elements of either operand
      auto xa = [](int atom) { return (W4 && SWAP) || WBF ? atom * (GEMM_BK / 2) : atom * GEMM_BK; };
      auto xb = [](int atom) { return (W4 && !SWAP) || WBF ? atom * (GEMM_BK / 2) : atom * GEMM_BK; };
      // No L2 prefetches run ahead of the ring: each prefetch request takes
      // the same copy engine as the loads, and without them the decode GEMMs
      // ran 8-9 % faster (measured at M = 1, 16 and 128).
      while (ok && sched.next(seg)) {
        int ta, tb;
        tile_coords(a, seg.tile, ta, tb);
        for (int kb = seg.kb0; kb < seg.kb1; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, SITE_PROD_EMPTY)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * SM::STAGE;
          mbar_arrive_expect_tx(&full[s], tx);
          // TSA: the stage's weights as boxes of 128 rows x 128 bytes (two
          // 64-element atoms of each row per box)
          if (TSA)
            for (int h = 0; h < KA / 2; ++h)
              tma_load_2d(st + h * (GEMM_BM * GEMM_BK), &tmA, &full[s], (kb * KA / 2 + h) * GEMM_BK,
                          ta * GEMM_BM, pol_a);
#pragma unroll
          for (int j = 0; j < KA; ++j) {
            // atoms past K read as zeros (TMA out-of-bounds fill) and add nothing
            const int atom = kb * KA + j;
            // a packed weight atom lands in the upper half of its slot
            if (!TSA)
              tma_load_2d(st + j * SM::A_ATOM + ((CONV && SWAP) ? SM::PACKED_OFF : 0), &tmA,
                          &full[s], xa(atom), ta * GEMM_BM, pol_a);
            tma_load_2d(st + SM::A_BYTES + j * SM::B_ATOM + ((CONV && !SWAP) ? SM::PACKED_OFF : 0),
                        &tmB, &full[s], xb(atom), tb * BN, pol_b);
          }
        }
      }
      // drain: make sure no copy is still landing in shared memory when the CTA exits
      const uint32_t n_issued = it;
      const uint32_t first = n_issued > static_cast<uint32_t>(S) ? n_issued - S : 0u;
      for (uint32_t j = first; j < n_issued; ++j) {
        int dummy = 0;
        volatile int* never = &dummy;
        mbar_wait(&full[j % S], (j / S) & 1u, never, SITE_DRAIN);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, local = 0;
      bool ok = true;
      while (ok && sched.next(seg)) {
        const uint32_t b = local & 1u;
        const uint32_t use = local >> 1;
        if (!mbar_wait(&tmem_empty[b], (use & 1u) ^ 1u, abort_flag, SITE_MMA_TMEM)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + b * SM::ACC_STRIDE;
        for (int kb = seg.kb0; kb < seg.kb1; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1u;
          if (!mbar_wait(CONV ? &conv[s] : &full[s], ph, abort_flag, SITE_MMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(smem + s * SM::STAGE);
          const uint32_t sb = sa + SM::A_BYTES;
          // TSA: this stage's expanded weights, 32 columns per K atom
          const uint32_t ta = tmem_base + SM::TSA_COL0 + (it % nbufs) * SM::TSA_COLS;
#pragma unroll
          for (int j = 0; j < SM::KA; ++j) {
#pragma unroll
            for (int k = 0; k < GEMM_BK / GEMM_UMMA_K; ++k) {
              const uint64_t bd = sw128_kmajor_desc(sb + j * SM::B_ATOM + k * GEMM_UMMA_K);
              const uint32_t acc = (kb > seg.kb0 || j > 0 || k > 0) ? 1u : 0u;
              if (TSA) {
                mma_bf16_ts(d, ta + j * (GEMM_BK / 4) + k * (GEMM_UMMA_K / 4), bd, IDESC, acc);
              } else {
                mma_s8(d, sw128_kmajor_desc(sa + j * SM::A_ATOM + k * GEMM_UMMA_K), bd, IDESC, acc);
              }
            }
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&tmem_full[b]);
        ++local;
      }
      // every MMA this thread issued must be complete before TMEM is released
      mma_commit(drain);
      int never = 0;
      mbar_wait(drain, 0u, &never, SITE_DRAIN);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int et = threadIdx.x - 64;  // 0..127 within the epilogue group
    uint32_t local = 0;
    uint32_t sync_phase = 0;
    // bounded rendezvous of the four epilogue warps (never an unbounded bar.sync)
    auto epi_rendezvous = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_sync);
      const bool r = mbar_wait(epi_sync, sync_phase & 1u, abort_flag, SITE_EPI_SYNC);
      ++sync_phase;
      __syncwarp();
      return r;
    };
    // output columns per staged 128-byte row (non-swap path)
    constexpr int OC = (EPI == EPI_BF16) ? 64 : 32;
    uint8_t* stage_buf = smem + SM::staging_offset(S) + q * 8192;
    int sbuf = 0;
    while (sched.next(seg)) {
      const uint32_t b = local & 1u;
      const uint32_t use = local >> 1;
      const bool got = mbar_wait(&tmem_full[b], use & 1u, abort_flag, SITE_EPI_FULL);
      __syncwarp();
      if (!got) break;
      tc_fence_after();
      int ta, tb;
      tile_coords(a, seg.tile, ta, tb);
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + b * SM::ACC_STRIDE;
      const int arow = ta * GEMM_BM + 32 * q + lane;  // operand-A row of this thread

      // A split tile: every contributing CTA adds its int32 partial into the
      // tile's accumulator (bulk reductions performed at L2); the CTA that
      // completes the tile's count reads it back, re-zeroes it and writes the
      // output.
      const int u_sk = seg.tile - a.dp_tiles;
      int32_t* acc_tile = a.ws_acc + static_cast<size_t>(u_sk) * (GEMM_BM * BN);
      if (seg.partial) {
#pragma unroll 1
        for (int c = 0; c < BN / CW; ++c) {
          uint32_t r[32];
          if (CW == 32) {
            tmem_ld_32x32b_x32(tbase + c * CW, r);
          } else {
            tmem_ld_32x32b_x16(tbase + c * CW, r);
          }
          tmem_ld_wait();
          if (lane == 0) bulk_wait_group_read<0>();  // the previous bulk op has read the buffer
          __syncwarp();
#pragma unroll
          for (int j4 = 0; j4 < CW / 4; ++j4)
            st_shared_v4(stage_buf + (j4 * 32 + lane) * 16, r[4 * j4], r[4 * j4 + 1], r[4 * j4 + 2],
                         r[4 * j4 + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (WBF)
              bulk_reduce_add_f32(acc_tile + (c * 4 + q) * 32 * CW, stage_buf, 128 * CW);
            else
              bulk_reduce_add_s32(acc_tile + (c * 4 + q) * 32 * CW, stage_buf, 128 * CW);
            bulk_commit_group();
          }
        }
      }
      bool finalize = !seg.partial;
      if (seg.partial) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tmem_empty[b]);
        if (lane == 0) {
          bulk_wait_group<0>();  // this warp's reductions are performed
          fence_proxy_async_global();
        }
        // the rendezvous orders every warp's performed reductions before the
        // counting thread's release below (one gpu-scope ordering point, not a
        // fence in every thread)
        __syncwarp();
        if (!epi_rendezvous()) break;
        if (et == 0) {
          const int c_lo = sk_owner(a, u_sk * a.num_kb);
          const int c_hi = sk_owner(a, (u_sk + 1) * a.num_kb - 1);
          const unsigned prev = atomic_add_acq_rel_gpu(&a.ws_counts[u_sk], 1u);
          const bool last = prev + 1u == static_cast<unsigned>(c_hi - c_lo + 1);
          if (last) a.ws_counts[u_sk] = 0u;  // leave the workspace clean for the next call
          *last_flag = last ? 1 : 0;
        }
        if (!epi_rendezvous()) break;
        // the counting thread acquired the other units' sums; the rendezvous
        // carries that to every thread of the CTA
        finalize = *last_flag != 0;
      }
      if (finalize) {
        if (!SWAP) {
          // ---- rows of the output tile: staged through shared memory, TMA stores
          const int m = arow;
          const int m0 = ta * GEMM_BM + 32 * q;
          float st = 0.f;
          if (EPI != EPI_S32 && m < a.M) st = WBF ? 1.0f : a.s_tok[m] * (W4 ? 0.0625f : 1.0f);
#pragma unroll 1
          for (int oc = 0; oc < (EPI == EPI_SWIGLU ? BN / 128 : 0); ++oc) {
            // MLP boundary: 128 accumulator columns (four blocks of 16 gate and
            // 16 up columns) give the 64 outputs of one staged 128-byte row
            uint8_t* buf = stage_buf + sbuf * 4096;
            if (lane == 0) bulk_wait_group_read<1>();  // the store from two chunks ago has read buf
            __syncwarp();
            const int sw = lane & 7;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              const int cc = oc * 4 + c;  // 32-column chunk of the tile
              uint32_t r[32];
              if (!seg.partial) {
                tmem_ld_32x32b_x32(tbase + cc * 32, r);
                tmem_ld_wait();
              } else {
                // the tile's sum; leave the accumulator at zero for the next call
                uint4* base = reinterpret_cast<uint4*>(acc_tile) + (cc * 4 + q) * 8 * 32 + lane;
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
              const int n0 = tb * BN + cc * 32;
              float sr[32];
#pragma unroll
              for (int j = 0; j < 32; ++j) sr[j] = n0 + j < a.N ? __ldg(a.s_row + n0 + j) : 0.f;
              uint32_t w[8];
              swiglu16(r, st, sr, w);
              st_shared_v4(buf + lane * 128 + (((2 * c) ^ sw) << 4), w[0], w[1], w[2], w[3]);
              st_shared_v4(buf + lane * 128 + (((2 * c + 1) ^ sw) << 4), w[4], w[5], w[6], w[7]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmY, buf, (tb * BN + oc * 128) / 2, m0);
              bulk_commit_group();
            }
            sbuf ^= 1;
          }
#pragma unroll 1
          for (int oc = 0; oc < (EPI == EPI_SWIGLU ? 0 : BN / OC); ++oc) {
            uint32_t r0[32], r1[32];
            if (!seg.partial) {
              tmem_ld_32x32b_x32(tbase + oc * OC, r0);
              if (OC == 64) tmem_ld_32x32b_x32(tbase + oc * OC + 32, r1);
              tmem_ld_wait();
            } else {
              // the tile's sum; leave the accumulator at zero for the next call
              const int c0 = oc * (OC / 32);
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
            uint8_t* buf = stage_buf + sbuf * 4096;
            if (lane == 0) bulk_wait_group_read<1>();  // the store from two chunks ago has read buf
            __syncwarp();
            const int sw = lane & 7;
            if (EPI == EPI_BF16) {
              const int n0 = tb * BN + oc * OC;
#pragma unroll
              for (int c16 = 0; c16 < 8; ++c16) {
                const uint32_t* rr = c16 < 4 ? r0 : r1;
                const int jb = (c16 & 3) * 8;
                const int n = n0 + c16 * 8;
                float sr[8];
                if (n < a.N) {
                  if (a.srow_vec) {
                    const float4 s0 = __ldg(reinterpret_cast<const float4*>(a.s_row + n));
                    const float4 s1 = __ldg(reinterpret_cast<const float4*>(a.s_row + n + 4));
                    sr[0] = s0.x; sr[1] = s0.y; sr[2] = s0.z; sr[3] = s0.w;
                    sr[4] = s1.x; sr[5] = s1.y; sr[6] = s1.z; sr[7] = s1.w;
                  } else {
#pragma unroll
                    for (int h = 0; h < 8; ++h) sr[h] = __ldg(a.s_row + n + h);
                  }
                } else {
#pragma unroll
                  for (int h = 0; h < 8; ++h) sr[h] = 0.f;
                }
                uint32_t w[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                  const float y0 = acc_value<WBF>(rr[jb + 2 * h]) * st * sr[2 * h];
                  const float y1 = acc_value<WBF>(rr[jb + 2 * h + 1]) * st * sr[2 * h + 1];
                  w[h] = pack_bf16x2(y0, y1);
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
              tma_store_2d(&tmY, buf, tb * BN + oc * OC, m0);
              bulk_commit_group();
            }
            sbuf ^= 1;
          }
        } else {
          // ---- swapped roles: lanes are weight rows n, columns are tokens m.
          // Each chunk of CW tokens is staged as [CW tokens][128 columns] (the
          // output's own layout) by the four warps, then one thread stores it
          // with TMA.  Chunks alternate between two 16 KB halves of the staging
          // area; before the warps meet after staging chunk k, the storing
          // thread waits until the store of chunk k - 1 has read its half, so
          // chunk k + 1 may overwrite it.
          constexpr int ES = (EPI == EPI_BF16) ? 2 : 4;
          const int n = arow;
          const int nl = 32 * q + lane;  // column of this lane in the staged tile
          float sr = 0.f;
          if (EPI != EPI_S32 && n < a.N) sr = a.s_row[n] * (W4 ? 0.0625f : 1.0f);
          bool staged_ok = true;
#pragma unroll 1
          for (int c = 0; c < BN / CW; ++c) {
            uint32_t r[32];
            if (!seg.partial) {
              if (CW == 32) {
                tmem_ld_32x32b_x32(tbase + c * CW, r);
              } else {
                tmem_ld_32x32b_x16(tbase + c * CW, r);
              }
              tmem_ld_wait();
            } else {
              uint4* base = reinterpret_cast<uint4*>(acc_tile) + (c * 4 + q) * (CW / 4) * 32 + lane;
              uint4 v[CW / 4];
#pragma unroll
              for (int j4 = 0; j4 < CW / 4; ++j4) v[j4] = __ldcg(base + j4 * 32);
              const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
              for (int j4 = 0; j4 < CW / 4; ++j4) {
                __stcg(base + j4 * 32, z);
                r[4 * j4] = v[j4].x;
                r[4 * j4 + 1] = v[j4].y;
                r[4 * j4 + 2] = v[j4].z;
                r[4 * j4 + 3] = v[j4].w;
              }
            }
            const int m0 = tb * BN + c * CW;
            uint8_t* xb = smem + SM::staging_offset(S) + sbuf * 16384;
            if (EPI == EPI_SWIGLU) {
              // MLP boundary, staged as [CW tokens][64 outputs]: each warp's
              // lanes are one block, gate rows in lanes 0-15 and the matching
              // up rows in lanes 16-31.  Of each token pair the low lanes form
              // the even token's outputs and the high lanes the odd token's.
              const bool upper = lane >= 16;
              const int col = 16 * q + (lane & 15);
#pragma unroll
              for (int j = 0; j < CW; j += 2) {
                const float st0 = m0 + j < a.M ? __ldg(a.s_tok + m0 + j) : 0.f;
                const float st1 = m0 + j + 1 < a.M ? __ldg(a.s_tok + m0 + j + 1) : 0.f;
                const float v0 = static_cast<float>(static_cast<int32_t>(r[j])) * st0 * sr;
                const float v1 = static_cast<float>(static_cast<int32_t>(r[j + 1])) * st1 * sr;
                const float other = __shfl_xor_sync(0xffffffffu, upper ? v0 : v1, 16);
                const float hv = upper ? silu_mul(other, v1) : silu_mul(v0, other);
                const __nv_bfloat16 hb = __float2bfloat16_rn(hv);
                asm volatile("st.shared.b16 [%0], %1;" ::"r"(smem_addr(xb + (j + (upper ? 1 : 0)) * 128 + col * 2)),
                             "h"(*reinterpret_cast<const unsigned short*>(&hb))
                             : "memory");
              }
            }
#pragma unroll
            for (int j = 0; j < (EPI == EPI_SWIGLU ? 0 : CW); ++j) {
              uint8_t* dst = xb + j * (128 * ES) + nl * ES;
              if (EPI == EPI_BF16) {
                const int m = m0 + j;
                const float st = m < a.M ? (WBF ? 1.0f : __ldg(a.s_tok + m)) : 0.f;
                const float v = acc_value<WBF>(r[j]) * st * sr;
                const __nv_bfloat16 hb = __float2bfloat16_rn(v);
                asm volatile("st.shared.b16 [%0], %1;" ::"r"(smem_addr(dst)),
                             "h"(*reinterpret_cast<const unsigned short*>(&hb))
                             : "memory");
              } else {
                asm volatile("st.shared.b32 [%0], %1;" ::"r"(smem_addr(dst)),
                             "r"(static_cast<uint32_t>(static_cast<int32_t>(r[j]) >> (W4 ? 4 : 0)))
                             : "memory");
              }
            }
            fence_proxy_async_smem();
            if (et == 0) bulk_wait_group_read<0>();  // the previous chunk's half has been read
            if (!epi_rendezvous()) {
              staged_ok = false;
              break;
            }
            if (et == 0) {
              // rows past M and columns past N are clipped by the store
              tma_store_2d(&tmY, xb, EPI == EPI_SWIGLU ? ta * GEMM_BM / 2 : ta * GEMM_BM, m0);
              bulk_commit_group();
            }
            sbuf ^= 1;
          }
          if (!staged_ok) break;
        }
      }
      if (!seg.partial) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tmem_empty[b]);
      }
      ++local;
    }
    // the staged outputs must have been read before the CTA exits; the global
    // writes themselves complete before the grid does
    if (lane == 0) bulk_wait_group_read<0>();
  } else if (TSA) {
    // ------------------------------------------------------------ int8 -> bf16
    // into tensor memory.  Warp w may access TMEM lanes 32 (w & 3) .. + 31:
    // lane l of it expands weight row 32 (w & 3) + l of the tile.  The stage's
    // rows landed in boxes of 128 bytes per row (atom j in box j / 2, chunks
    // 4 (j & 1) .. + 3) with the 128-byte swizzle (16-byte chunk c of row r at
    // chunk c ^ (r & 7)), so each quarter-warp's 16-byte loads fall in eight
    // different bank groups.
    const int q = warp & 3;
    const int r = 32 * q + lane;
    const uint32_t tlane = static_cast<uint32_t>(32 * q) << 16;
    const int rsw = r & 7;
    uint32_t it = 0;
    bool ok = true;
    while (ok && sched.next(seg)) {
      for (int kb = seg.kb0; kb < seg.kb1; ++kb, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1u;
        if (!mbar_wait(&full[s], ph, abort_flag, SITE_CONV_FULL)) {
          ok = false;
          break;
        }
        const int x = static_cast<int>(it % static_cast<uint32_t>(nbufs));
        if (it >= static_cast<uint32_t>(nbufs)) {
          // buffer x last held stage it - nbufs: its MMAs are complete once that
          // stage's slot was released (the release after it needs this stage's
          // MMAs, so the parity is unambiguous)
          const uint32_t prev = it - static_cast<uint32_t>(nbufs);
          if (!mbar_wait(&empty[prev % S], (prev / S) & 1u, abort_flag, SITE_CONV_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        const uint8_t* st = smem + s * SM::STAGE;
        const uint32_t ta = tmem_base + tlane + SM::TSA_COL0 + x * SM::TSA_COLS;
#pragma unroll
        for (int j = 0; j < SM::KA; ++j) {
          const uint8_t* row = st + (j >> 1) * (GEMM_BM * GEMM_BK) + r * GEMM_BK;
          uint32_t o[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 pk = ld_shared_v4(row + (((4 * (j & 1) + c) ^ rsw) << 4));
            i8x4_to_bf16x4(pk.x, o[8 * c], o[8 * c + 1]);
            i8x4_to_bf16x4(pk.y, o[8 * c + 2], o[8 * c + 3]);
            i8x4_to_bf16x4(pk.z, o[8 * c + 4], o[8 * c + 5]);
            i8x4_to_bf16x4(pk.w, o[8 * c + 6], o[8 * c + 7]);
          }
          tmem_st_32x32b_x32(ta + j * (GEMM_BK / 4), o);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&conv[s]);
      }
    }
  } else if (CONV) {
    // ------------------------------------------------------------ int4 unpack
    // Each thread reads its share of every packed atom of the stage, the four
    // warps meet (bounded), then each writes the expanded swizzled rows over
    // the slot the packed bytes came in.
    const int ct = threadIdx.x - 192;  // 0..127
    constexpr int WR = SM::W_ROWS;
    constexpr int PER = WR * 4 / 128;  // 16-byte packed pieces per thread and atom
    uint32_t it = 0, cv_phase = 0;
    bool ok = true;
    while (ok && sched.next(seg)) {
      for (int kb = seg.kb0; kb < seg.kb1; ++kb, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1u;
        if (!mbar_wait(&full[s], ph, abort_flag, SITE_CONV_FULL)) {
          ok = false;
          break;
        }
        uint8_t* st = smem + s * SM::STAGE;
        uint4 pks[SM::KA][PER];
#pragma unroll
        for (int j = 0; j < SM::KA; ++j) {
          const uint8_t* packed =
              (SWAP ? st + j * SM::A_ATOM : st + SM::A_BYTES + j * SM::B_ATOM) + SM::PACKED_OFF;
#pragma unroll
          for (int i = 0; i < PER; ++i) {
            const int idx = ct + 128 * i;
            // explicit shared-memory loads and stores schedule better for the
            // 256-row tiles, generic ones for the decode tiles (measured)
            const uint8_t* src = packed + (idx >> 2) * 64 + (idx & 3) * 16;
            pks[j][i] = SWAP ? *reinterpret_cast<const uint4*>(src) : ld_shared_v4(src);
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
        uint8_t* unp = SWAP ? st + j * SM::A_ATOM : st + SM::A_BYTES + j * SM::B_ATOM;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const int idx = ct + 128 * i;
          const int r = idx >> 2, pc = idx & 3;
          const uint4 pk = pks[j][i];
          const uint32_t w[4] = {pk.x, pk.y, pk.z, pk.w};
          uint32_t o[8];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const uint32_t lo = (w[h] << 4) & 0xF0F0F0F0u;
            const uint32_t hi = w[h] & 0xF0F0F0F0u;
            o[2 * h] = __byte_perm(lo, hi, 0x5140);
            o[2 * h + 1] = __byte_perm(lo, hi, 0x7362);
          }
          const int sw = r & 7;
          uint8_t* d0 = unp + r * 128 + (((2 * pc) ^ sw) << 4);
          uint8_t* d1 = unp + r * 128 + (((2 * pc + 1) ^ sw) << 4);
          if (SWAP) {
            *reinterpret_cast<uint4*>(d0) = make_uint4(o[0], o[1], o[2], o[3]);
            *reinterpret_cast<uint4*>(d1) = make_uint4(o[4], o[5], o[6], o[7]);
          } else {
            st_shared_v4(d0, o[0], o[1], o[2], o[3]);
            st_shared_v4(d1, o[4], o[5], o[6], o[7]);
          }
        }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&conv[s]);
      }
    }
  }

  __syncwarp();  // roles ran on single lanes: reconverge before the aligned barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, SM::TMEM_COLS);
  }
}

}  // namespace convrot
