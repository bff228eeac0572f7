// Per-token activation rotate-quantise for the hot path:
// [RMSNorm with the (1 + w) weight] -> group Hadamard (FWHT-256 or -16) ->
// per-token absmax -> int8 codes and one fp32 scale per token
// ("MOSS-Image Qwen3.5-9B text encoder, INT8 (W8A8, ConvRot)", file table,
// "Matmul" row: the input is rotated by the same Hadamard as the weight and
// rounded to int8 per token; "Changed" row and "How it was made": the fp32
// RMSNorm weight carries the folded SmoothQuant scale).
//
// Work split.  One CTA per SM; every warp is a consumer.  Stages of R
// consecutive token rows stream into a shared-memory ring, one TMA copy per
// stage of a [R rows][K / 64 lines][64 elements] box with the 128-byte
// swizzle: thread 0 fills the ring at the start, and afterwards the warp that
// releases a slot last (a shared counter per slot) refills it with the unit
// `stages` steps later (and, with the norm, prefetches the one after into
// L2).  No warp is set aside for the copies: a CTA of 24 warps gets up to 80
// registers per thread, one of 32 warps (for teams whose width in warps
// divides 32) up to 64.  The fp32 norm weight is copied once per CTA the same
// way, as lines of 32 values.  The swizzle (16-byte chunk c of 128-byte line
// r stored at chunk c ^ (r & 7)) puts the eight threads of a
// group, which read 64 bytes of the row (and 128 bytes of the weight) each,
// in eight different bank groups.
// The consumer warps form R teams, one row each; a row's 256-element groups
// are taken by eight threads, 32 elements each.  Every thread keeps its
// elements in sixteen packed fp32 pairs (f32x2 registers).
//
// Element e of a 256-group (bits e7..e0) moves through two register layouts:
//  * phase 1: thread l (0..7) holds e7..e5 = l and all of e4..e0; pair k of
//    its sixteen holds e0 = 0 / 1 in its two halves and e4..e1 = k;
//  * phase 2: thread l holds e4..e2 = l and all of e7..e5 and e1..e0; chunk t
//    (pairs 2t, 2t + 1) holds e7..e5 = t.
// The butterfly of e0 is taken while the bf16 inputs are unpacked (scalar
// add and subtract of the two halves of each 32-bit word); e1..e4 are
// butterflies between pairs in phase 1 and e5..e7 in phase 2, each one packed
// add and one packed subtract per four elements.  Between the phases the
// eight threads of a group swap 16-byte chunks (four consecutive elements)
// through shared memory: eight stores and eight loads per thread, at
// positions that put the eight stores (and the eight loads) of one
// quarter-warp in eight different 16-byte bank groups.  Half of the 1 KB a
// group needs is the group's own 512 bytes of the staged input row, which is
// free once its eight threads have loaded it; the stage is released to the
// producer after the exchange.  A 16-point group only needs phase 1.
//
// Per-row scalars: the 1/16 (or 1/4) of the normalised Hadamard and the
// RMSNorm factor r do not change the codes (they depend on v / max|v| only),
// so they enter only the fp64 computation of the per-row scale.  Codes are
// rint(v * 127 / max|v|) with round-half-even, taken in one rounding by
// fma(v, inv, 1.5 * 2^23) (the integer lands in the low mantissa bits; its low
// byte is the two's-complement code).
#pragma once

#include "ptx.cuh"

namespace convrot {

constexpr int AQ_MAX_STAGES = 8;
constexpr int AQ_MAX_CWARPS = 32;      // warps per CTA, all consumers (24 or 32 per launch)
constexpr int AQ_MAX_TEAM_WARPS = 16;  // a row of up to 16384 elements
constexpr int AQ_MAX_SLOTS = 15;       // rows per stage for teams wider than a warp (barriers 1..15)
constexpr int AQ_XPOSE_WARP_BYTES = 2048;  // exchange halves: four groups x 512 bytes
constexpr int AQ_SMEM_BUDGET = 214 * 1024;  // dynamic; the static arrays take ~11 KB more
constexpr int AQ_MAX_RINGS = 32;       // staging groups per CTA (a team, or a warp of narrow teams)

struct ActArgs {
  const uint16_t* x;    // [M, K] bf16 bits (L2 prefetch and the rare fp64 path)
  int8_t* xq;           // [M, K]
  float* s_tok;         // [M]
  int M, K;
  float eps;
  int team;        // threads per row: 8 per (virtual) 256-element group, padded
  int rows;        // rows per unit = teams per CTA
  int group_rows;  // rows per staging group: 1 for teams of whole warps, 32 / team below
  int stages;      // ring slots per staging group
  int slot_stride; // bytes between ring slots: group_rows * K * 2 rounded up to 1024
  int w_box_lines;   // 128-byte lines of the norm weight per copy
  int w_copies;      // copies of w_box_lines lines (0 without a norm)
  int wsm_bytes;     // shared bytes of the norm weight (all copies, rounded up to 1024) or 0
  int xpose_bytes;  // shared bytes of the groups' own exchange halves (consumer warps x 2048) or 0
};

// Packed fp32x2 arithmetic: one instruction for the two halves of a 64-bit register.
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  return static_cast<uint64_t>(__float_as_uint(lo)) |
         (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ uint64_t u2_pack(uint32_t lo, uint32_t hi) {
  return static_cast<uint64_t>(lo) | (static_cast<uint64_t>(hi) << 32);
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float f2_hi(uint64_t v) {
  return __uint_as_float(static_cast<uint32_t>(v >> 32));
}

__device__ __forceinline__ void st_v4_global(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// The sixteen pairs of a thread; chunk c (the unit the exchange moves) is
// pairs 2c and 2c + 1.
typedef uint64_t AqRegs[16];

__device__ __forceinline__ uint64_t& aq_pair(AqRegs& q, int k) { return q[k]; }

// Butterfly between the pairs k and k ^ D (all sixteen, in place).
template <int D>
__device__ __forceinline__ void aq_stage(AqRegs& q) {
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    if (!(k & D)) {
      const uint64_t a = aq_pair(q, k), b = aq_pair(q, k | D);
      aq_pair(q, k) = f2_add(a, b);
      aq_pair(q, k | D) = f2_sub(a, b);
    }
  }
}

// Phase-1 load of the thread's 32 elements from the staged row: four 16-byte
// loads of eight bf16 values; load m reads elements e0 + 8m .. e0 + 8m + 7
// into pairs 4m .. 4m + 3.  With NORM, sum(x^2) of the raw inputs is
// accumulated (a product and three fused adds per element half, then a
// pairwise sum) and x is multiplied by 1 + w as x + x w (one rounding of the
// exact product).  With a transform, the butterfly of element bit 0 is taken
// here on the two halves of every 32-bit word.
// x0 + x1 and x1 - x0 of the two bf16 halves of w, x0 given in fp32: the
// high half enters the fp32 add as bf16 (mixed-precision add), which saves
// unpacking it.  One rounding each, the same as two fp32 adds.
__device__ __forceinline__ uint64_t aq_bf16_butterfly(uint32_t w, float x0) {
  float s, d;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "add.rn.f32.bf16 %0, hi, %3;\n\tsub.rn.f32.bf16 %1, hi, %3;\n\t}"
      : "=f"(s), "=f"(d)
      : "r"(w), "f"(x0));
  return f2_pack(s, d);
}

// Phase-1 load of the thread's 32 elements from the staged row: four 16-byte
// loads of eight bf16 values; load m reads elements e0 + 8m .. e0 + 8m + 7
// into pairs 4m .. 4m + 3.  The swizzled copy puts piece m of the thread at
// shared address xaddr ^ 16m (and chunk j of its norm weight at waddr ^ 16j):
// the caller passes the addresses of piece 0.  With NORM, sum(x^2) of the raw
// inputs is accumulated (a product and three fused adds per element half,
// then a pairwise sum) and x is multiplied by 1 + w as x + x w (one rounding
// of the exact product).  With a transform, the butterfly of element bit 0 is
// taken here on the two halves of every 32-bit word; without the norm its
// difference half comes out as x1 - x0, i.e. every element with bit 0 set is
// negated, which the caller undoes in the quantisation scale.
template <int GRP, bool NORM, bool WHOLE>
__device__ __forceinline__ void aq_load(uint32_t xaddr, uint32_t waddr, int K, int e0, bool ok,
                                        AqRegs& q, float& sq) {
  uint64_t acc01 = 0, acc23 = 0;  // pairwise: (load 0 + load 1) + (load 2 + load 3)
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int e = e0 + 8 * m;
    // whole groups: every address is inside the staged row (the caller points
    // threads of padding groups at a real group and discards their values)
    const bool in = WHOLE ? true : (ok && e < K);
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    if (in) raw = lds128(xaddr ^ (16u * m));
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint4 n0 = make_uint4(0u, 0u, 0u, 0u), n1 = n0;
    if (NORM && in) {
      n0 = lds128(waddr ^ (32u * m));
      n1 = lds128(waddr ^ (32u * m + 16u));
    }
    const uint64_t wn[4] = {u2_pack(n0.x, n0.y), u2_pack(n0.z, n0.w), u2_pack(n1.x, n1.y),
                            u2_pack(n1.z, n1.w)};
    uint64_t part = 0;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float x0 = __uint_as_float(w[h] << 16);
      if (NORM) {
        const uint64_t xx = f2_pack(x0, __uint_as_float(w[h] & 0xFFFF0000u));
        part = h == 0 ? f2_mul(xx, xx) : f2_fma(xx, xx, part);
        const uint64_t y = f2_fma(xx, wn[h], xx);
        const float y0 = f2_lo(y), y1 = f2_hi(y);
        aq_pair(q, 4 * m + h) = GRP ? f2_pack(y0 + y1, y0 - y1) : y;
      } else if (GRP) {
        aq_pair(q, 4 * m + h) = aq_bf16_butterfly(w[h], x0);
      } else {
        aq_pair(q, 4 * m + h) = f2_pack(x0, __uint_as_float(w[h] & 0xFFFF0000u));
      }
    }
    if (NORM) {
      if (m == 0) acc01 = part;
      else if (m == 1) acc01 = f2_add(acc01, part);
      else if (m == 2) acc23 = part;
      else acc23 = f2_add(acc23, part);
    }
  }
  if (NORM) {
    const uint64_t s = f2_add(acc01, acc23);
    sq += f2_lo(s) + f2_hi(s);
  }
}

// Phase 1 -> phase 2 for 256-point groups.  Thread l stores its chunk c
// (pairs 2c, 2c + 1: elements 32 l + 4c .. + 3) at position 8 (c & 3) +
// (l ^ c) of area a (c < 4) or b (c >= 4); thread l then loads chunk l of
// every thread a from position 8 (l & 3) + (a ^ l) of area a (l < 4) or b
// into its chunk a.  Each store step c and each load step a touches bank
// group (l ^ c) or (a ^ l): eight different ones over the group's threads.
// The areas are 512-byte aligned, so with A = area a + 16 l and B = area b +
// 16 l the store address is (A or B) ^ 16c, plus 128 (c & 3), and with R =
// (area a or b) + 128 (l & 3) + 16 l the load address is R ^ 16a.  Every lane
// of the warp calls this (it synchronises the warp).  A padding group past
// the end of the row passes its own area b as area a too: it moves values
// nobody reads, without touching the staged row.
__device__ __forceinline__ void aq_exchange(AqRegs& q, uint32_t A, uint32_t B, uint32_t R) {
  __syncwarp();  // the group's inputs (area a) and the last exchange (area b) are read
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    sts128(((c < 4 ? A : B) ^ (16u * c)) + 128u * (c & 3), static_cast<uint32_t>(q[2 * c]),
           static_cast<uint32_t>(q[2 * c] >> 32), static_cast<uint32_t>(q[2 * c + 1]),
           static_cast<uint32_t>(q[2 * c + 1] >> 32));
  }
  __syncwarp();
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const uint4 v = lds128(R ^ (16u * a));
    q[2 * a] = u2_pack(v.x, v.y);
    q[2 * a + 1] = u2_pack(v.z, v.w);
  }
}

__device__ __forceinline__ float aq_absmax(const AqRegs& q) {
  float m0 = 0.f, m1 = 0.f, m2 = 0.f, m3 = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    m0 = fmaxf(m0, fabsf(f2_lo(q[2 * c])));
    m1 = fmaxf(m1, fabsf(f2_hi(q[2 * c])));
    m2 = fmaxf(m2, fabsf(f2_lo(q[2 * c + 1])));
    m3 = fmaxf(m3, fabsf(f2_hi(q[2 * c + 1])));
  }
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

// Four codes (the low bytes of four rounded values) in one word.
__device__ __forceinline__ uint32_t aq_pack4(uint64_t a, uint64_t b) {
  const uint32_t lo = __byte_perm(static_cast<uint32_t>(a), static_cast<uint32_t>(a >> 32), 0x0040);
  const uint32_t hi = __byte_perm(static_cast<uint32_t>(b), static_cast<uint32_t>(b >> 32), 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

// Reductions over the threads of one row team.  Teams narrower than a warp
// are aligned power-of-two lane ranges and reduce with shuffles.  Teams of
// whole warps take the warp maximum with one redux (max|v| is non-negative, so
// its bit pattern orders like an unsigned integer) and the fp64 sum with a
// fixed shuffle tree; warps of a wider team then meet at an mbarrier of their
// row slot (a bounded wait) and every lane combines the warps' partials the
// same way, read lane-parallel from shared buffers that alternate between two
// halves: a warp reuses a half only after every warp of the team has arrived
// for the use in between, i.e. has finished reading it.  Every warp of a team
// combines the same values in the same order, so the results agree bit for
// bit.  Returns false if the rendezvous gave up (abort or timeout).
struct AqReducer {
  float* smax;    // [2][AQ_MAX_SLOTS][AQ_MAX_TEAM_WARPS]
  double* ssum;   // [2][AQ_MAX_SLOTS][AQ_MAX_TEAM_WARPS]
  uint64_t* bar;  // the row slot's rendezvous (arrival count: warps of the team)
  volatile int* abort;
  int team, slot, lane, warp_in_team, nwarps;
  uint32_t parity;

  template <bool WIDE, bool SUM>
  __device__ __forceinline__ bool reduce(float& mx, double& sm) {
    if (!WIDE) {
      for (int o = team >> 1; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (SUM) sm += __shfl_xor_sync(0xffffffffu, sm, o);
      }
      return true;
    }
    mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mx)));
    if (SUM) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
    }
    if (nwarps == 1) return true;
    const int base = (static_cast<int>(parity) * AQ_MAX_SLOTS + slot) * AQ_MAX_TEAM_WARPS;
    if (lane == 0) {
      smax[base + warp_in_team] = mx;
      if (SUM) ssum[base + warp_in_team] = sm;
      mbar_arrive(bar);
    }
    const bool met = mbar_wait_spin(bar, parity, abort, SITE_EPI_SYNC);
    __syncwarp();
    parity ^= 1u;
    if (!__all_sync(0xffffffffu, met)) return false;
    const bool have = lane < nwarps;
    const float pm = have ? smax[base + lane] : 0.f;
    mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(pm)));
    if (SUM) {
      // every lane sums all 32 (lanes past the team's warps hold 0)
      double ps = have ? ssum[base + lane] : 0.0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      sm = ps;
    }
    return true;
  }
};

// fp64 sum of squares of the raw inputs of the thread's 32 elements, read
// from global memory (the rare path for rows whose fp32 sum of squares leaves
// the safe range: |x| beyond ~1e18, or tiny rows).
__device__ __forceinline__ double aq_sumsq64(const uint16_t* grow, int K, int e0, bool ok) {
  double acc = 0.0;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int e = e0 + 8 * m;
    if (ok && e < K) {
      const uint4 raw = *reinterpret_cast<const uint4*>(grow + e);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const double lo = static_cast<double>(__uint_as_float(w[h] << 16));
        const double hi = static_cast<double>(__uint_as_float(w[h] & 0xFFFF0000u));
        acc = fma(lo, lo, acc);
        acc = fma(hi, hi, acc);
      }
    }
  }
  return acc;
}

template <int GRP>
__host__ __device__ constexpr double aq_group_norm() {
  return GRP == 256 ? 1.0 / 16.0 : (GRP == 16 ? 1.0 / 4.0 : 1.0);
}

// Issues the copy of the RG rows of group q in unit u (rows u R + q RG ..)
// into one slot of the group's ring; rows past M read as zeros and the box
// always delivers RG * K * 2 bytes.  Counts the copy for the exit drain.
__device__ __forceinline__ void aq_issue(const CUtensorMap* tmX, const ActArgs& a, uint8_t* slot,
                                         uint64_t* bar, unsigned* count, int u, int q) {
  mbar_arrive_expect_tx(bar, static_cast<uint32_t>(a.group_rows) * a.K * 2u);
  tma_load_3d(slot, tmX, bar, 0, 0, u * a.rows + q * a.group_rows);
  ++*count;
}

__device__ __forceinline__ void aq_prefetch(const ActArgs& a, int u, int q) {
  const int r0 = u * a.rows + q * a.group_rows;
  if (r0 < a.M)
    bulk_prefetch_l2(a.x + static_cast<size_t>(r0) * a.K,
                     static_cast<uint32_t>(min(a.group_rows, a.M - r0)) * a.K * 2);
}

// WIDE: the team is one or more whole warps (K >= 1024).  NW: warps per CTA,
// 24 (up to 80 registers per thread) or 32 (up to 64), chosen by the host for
// teams whose width divides it.
template <int GRP, bool NORM, bool WIDE, int NW>
__global__ void __launch_bounds__(32 * NW, 1)
    actquant_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    ActArgs a) {
  static_assert(GRP == 0 || GRP == 16 || GRP == 256, "group size 0, 16 or 256");
  // L2 prefetch of the unit after the ring's next one.  Without the norm it
  // only takes the copy engine from the ring's own copies (measured without
  // it: 8192 x 4096 24.0 -> 23.0 us); with the norm, dropping it costs the
  // 32-warp build registers (more spills) and 4 % at 2048 x 4096, so it stays.
  constexpr bool AQ_L2_PREFETCH = NORM;
  // K is a multiple of 256 with 256-point groups: no per-element bounds checks
  constexpr bool WHOLE = GRP == 256;
  pdl_launch_dependents();  // the grid is co-resident: dependents only take idle SMs
  __shared__ float s_max[2 * AQ_MAX_SLOTS * AQ_MAX_TEAM_WARPS];
  __shared__ double s_sum[2 * AQ_MAX_SLOTS * AQ_MAX_TEAM_WARPS];
  __shared__ uint64_t full[AQ_MAX_RINGS * AQ_MAX_STAGES], wbar, tbar[AQ_MAX_SLOTS];
  __shared__ unsigned released[AQ_MAX_RINGS * AQ_MAX_STAGES], issued[AQ_MAX_RINGS * AQ_MAX_STAGES];
  __shared__ int abort_word;
  extern __shared__ __align__(1024) uint8_t aq_smem_raw[];
  // the swizzled copies need 1024-byte aligned destinations
  uint8_t* aq_smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(aq_smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
  uint8_t* wsm = aq_smem;
  uint8_t* xpose = aq_smem + a.wsm_bytes;
  uint8_t* rings = xpose + a.xpose_bytes;
  const int lines = a.K >> 6;  // 128-byte lines of one staged row
  volatile int* abort_flag = &abort_word;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int gwarps = WIDE ? (a.team >> 5) : 1;  // warps of one staging group
  const int ngroups = (a.team * a.rows) / (32 * gwarps);
  const int units = (a.M + a.rows - 1) / a.rows;
  if (threadIdx.x == 0) {
    for (int j = 0; j < ngroups * a.stages; ++j) {
      mbar_init(&full[j], 1);
      released[j] = 0u;
      issued[j] = 0u;
    }
    mbar_init(&wbar, 1);
    // team rendezvous: one arrival per warp of a team wider than a warp
    if (a.team > 32)
      for (int r = 0; r < a.rows; ++r) mbar_init(&tbar[r], static_cast<uint32_t>(a.team >> 5));
    abort_word = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmX);
    if (NORM) tma_prefetch_desc(&tmW);
  }
  __syncthreads();
  pdl_wait();  // x, w, Xq and s_tok may belong to the previous kernel
  if (threadIdx.x == 0) {
    if (NORM) {
      // the norm weight [K] fp32, copied once per CTA next to the first rows
      mbar_arrive_expect_tx(&wbar, static_cast<uint32_t>(a.w_copies * a.w_box_lines) * 128u);
      for (int c = 0; c < a.w_copies; ++c)
        tma_load_2d_plain(wsm + c * a.w_box_lines * 128, &tmW, &wbar, 0, c * a.w_box_lines);
    }
    // fill every group's ring, then warm L2 with each group's next unit
    for (int j = 0; j < a.stages; ++j) {
      const int u = blockIdx.x + j * gridDim.x;
      if (u >= units) break;
      for (int q = 0; q < ngroups; ++q)
        aq_issue(&tmX, a, rings + (q * a.stages + j) * a.slot_stride, &full[q * a.stages + j],
                 &issued[q * a.stages + j], u, q);
    }
    const int uf = blockIdx.x + a.stages * gridDim.x;
    if (AQ_L2_PREFETCH && uf < units)
      for (int q = 0; q < ngroups; ++q) aq_prefetch(a, uf, q);
  }
  // ------------------------------------------------------------ consumers
  const int ct = threadIdx.x;
  const int slot = ct / a.team;           // row of the unit
  const int t = ct - slot * a.team;
  const int q = warp / gwarps;            // staging group
  const int rq = slot - q * a.group_rows; // row within the group's copy
  const int G = (a.K + 255) >> 8;
  const int g = t >> 3;  // (virtual) 256-element group of the row
  const int l = t & 7;   // thread of the group
  const bool gok = g < G;
  // padding groups of a whole-group team read a real group's row and drop it
  const int gl = WHOLE ? min(g, G - 1) : g;
  const int e0 = g * 256 + 32 * l;  // the thread's phase-1 elements: e0 .. e0 + 31
  const int xline = rq * lines + 4 * gl + (l >> 1);  // the line holding its 64 bytes of the row
  const int aline = rq * lines + 4 * g;              // the group's four lines (exchange area a)
  // shared addresses relative to a ring slot: piece 0 of the thread's
  // elements in the swizzled row (line xline, chunk 4 (l & 1) ^ (xline & 7)),
  // and the group's exchange areas (see aq_exchange)
  const uint32_t xoff = static_cast<uint32_t>(xline * 128 + 16 * ((4 * (l & 1)) ^ (xline & 7)));
  const uint32_t waddr = smem_addr(wsm) + static_cast<uint32_t>((8 * gl + l) * 128 + 16 * l);
  const uint32_t area_b = smem_addr(xpose) + static_cast<uint32_t>(warp * AQ_XPOSE_WARP_BYTES +
                                                                    (lane >> 3) * 512);
  const uint32_t xB = area_b + 16u * l;
  uint8_t* ring = rings + q * a.stages * a.slot_stride;
  uint64_t* qfull = full + q * a.stages;
  unsigned* qrel = released + q * a.stages;
  unsigned* qiss = issued + q * a.stages;
  // the warp of the group that releases a ring slot last refills it with the
  // group's rows `stages` units later (and may warm L2 with the unit after that)
  auto release = [&](int s, int u) {
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      if (atomicAdd(&qrel[s], 1u) == static_cast<unsigned>(gwarps - 1)) {
        qrel[s] = 0u;
        __threadfence_block();
        const int un = u + a.stages * static_cast<int>(gridDim.x);
        if (un < units) aq_issue(&tmX, a, ring + s * a.slot_stride, &qfull[s], &qiss[s], un, q);
        const int uf = un + static_cast<int>(gridDim.x);
        if (AQ_L2_PREFETCH && uf < units) aq_prefetch(a, uf, q);
      }
    }
  };
  AqReducer red{s_max, s_sum, &tbar[slot < AQ_MAX_SLOTS ? slot : 0], abort_flag, a.team, slot, lane,
                t >> 5, a.team >> 5, 0u};
  const bool alive = !NORM || mbar_wait(&wbar, 0u, abort_flag, SITE_EPI_FULL);
  int s = 0;
  uint32_t ph = 0;
  for (int u = blockIdx.x; alive && u < units; u += gridDim.x) {
    // every warp of a team waits on the same barrier (it completes for all or
    // none; an abort is CTA-wide), so the team reductions stay matched
    if (!mbar_wait_spin(&qfull[s], ph, abort_flag, SITE_EPI_FULL)) break;
    const int row = u * a.rows + slot;
    const bool row_ok = row < a.M;
    const bool ok = row_ok && gok;
    const uint32_t stage = smem_addr(ring) + static_cast<uint32_t>(s * a.slot_stride);
    AqRegs p;
    float sq = 0.f;
    aq_load<GRP, NORM, WHOLE>(stage + xoff, waddr, a.K, e0, ok, p, sq);
    if (GRP != 256) release(s, u);  // slot read
    if (GRP) {
      aq_stage<1>(p);  // element bit 1
      aq_stage<2>(p);  // bit 2
      aq_stage<4>(p);  // bit 3
    }
    if (GRP == 256) {
      aq_stage<8>(p);  // bit 4
      // half of the exchange area is the group's 512 bytes (four lines) of the staged row
      const uint32_t xA = gok ? stage + static_cast<uint32_t>(aline * 128) + 16u * l : xB;
      aq_exchange(p, xA, xB, (l < 4 ? xA : xB) + 128u * (l & 3));
      // the row's ring slot was written by this thread: order those writes
      // before the copy that will refill the slot, then release it
      fence_proxy_async_smem();
      release(s, u);
      aq_stage<2>(p);  // bit 5
      aq_stage<4>(p);  // bit 6
      aq_stage<8>(p);  // bit 7
    }
    if (++s == a.stages) {
      s = 0;
      ph ^= 1u;
    }
    float amax = gok ? aq_absmax(p) : 0.f;
    double sumsq = static_cast<double>(gok ? sq : 0.f);
    if (!red.reduce<WIDE, NORM>(amax, sumsq)) break;
    if (NORM) {
      // Rows whose fp32 sum of squares left the safe range (|x| above ~1e18,
      // or tiny rows) take an fp64 recompute.  The decision is team-uniform
      // (reduced values), and made warp-wide so that every shuffle converges.
      const bool need = amax > 0.f && !(sumsq > 0x1p-100 && sumsq < 0x1p+100);
      if (__any_sync(0xffffffffu, need)) {
        const uint16_t* grow = a.x + static_cast<size_t>(row_ok ? row : 0) * a.K;
        double s64 = aq_sumsq64(grow, a.K, e0, ok);
        float dummy = 0.f;
        if (!red.reduce<WIDE, true>(dummy, s64)) break;
        if (need) sumsq = s64;
      }
    }
    const float inv = amax > 0.f ? 127.0f / amax : 0.0f;
    // codes: rint(v * inv) in one rounding (low byte of v * inv + 1.5 * 2^23);
    // without the norm, the odd elements of a transform arrive negated
    const uint64_t inv2 = f2_pack(inv, (GRP && !NORM) ? -inv : inv);
    const uint64_t mag2 = f2_pack(12582912.0f, 12582912.0f);
#pragma unroll
    for (int k = 0; k < 16; ++k) p[k] = f2_fma(p[k], inv2, mag2);
    int8_t* qrow = a.xq + static_cast<size_t>(row_ok ? row : 0) * a.K;
    if (GRP == 256) {
      // chunk t: elements 32 t + 4 l + 0..3 of the group (predicated stores)
      int8_t* qp = qrow + e0 - 28 * l;  // g * 256 + 4 l
      const uint32_t on = ok ? 1u : 0u;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t w = aq_pack4(p[2 * c], p[2 * c + 1]);
        asm volatile("{\n\t.reg .pred pq;\n\tsetp.ne.u32 pq, %2, 0;\n\t@pq st.global.u32 [%0], %1;\n\t}"
                     ::"l"(qp + 32 * c), "r"(w), "r"(on) : "memory");
      }
    } else {
      // chunk c: elements e0 + 4c + 0..3; sixteen codes per 16-byte store
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int e = e0 + 16 * h;
        if (ok && e < a.K) {
          st_v4_global(qrow + e, aq_pack4(p[8 * h], p[8 * h + 1]), aq_pack4(p[8 * h + 2], p[8 * h + 3]),
                       aq_pack4(p[8 * h + 4], p[8 * h + 5]), aq_pack4(p[8 * h + 6], p[8 * h + 7]));
        }
      }
    }
    if (row_ok && t == 0) {
      // the per-row scale, needed by one thread only: max|v| times the 1/16
      // (1/4) of the normalised Hadamard and, with the norm, r = (mean x^2 +
      // eps)^-1/2 in fp64; without the norm amax times that power of two,
      // divided by 127 with one rounding
      float sc = 0.f;
      if (amax > 0.f) {
        if (NORM) {
          const double r = 1.0 / sqrt(sumsq / static_cast<double>(a.K) + static_cast<double>(a.eps));
          sc = static_cast<float>(static_cast<double>(amax) * aq_group_norm<GRP>() * r / 127.0);
        } else {
          sc = __fdiv_rn(amax * static_cast<float>(aq_group_norm<GRP>()), 127.0f);
        }
      }
      a.s_tok[row] = sc;
    }
  }
  // After an abort, copies may still be landing in this CTA's rings: wait
  // (bounded) for the last copy issued into every slot before exiting.
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    int dummy = 0;
    for (int j = 0; j < ngroups * a.stages; ++j)
      if (issued[j]) mbar_wait(&full[j], (issued[j] - 1u) & 1u, &dummy, SITE_DRAIN);
    if (NORM) mbar_wait(&wbar, 0u, &dummy, SITE_DRAIN);
  }
}

}  // namespace convrot
