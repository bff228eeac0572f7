// Row-wise ConvRot quantisation kernels: [RMSNorm | column scale] -> group
// Hadamard (FWHT-256) -> per-row absmax -> int8 codes (or int4 codes with a
// per-row clip search).
//
// One kernel family serves three entry points:
//  * activations (per token): optional fused RMSNorm with the (1 + w) weight
//    ("MOSS-Image Qwen3.5-9B text encoder, INT8 (W8A8, ConvRot)", file table,
//    "Matmul" and "Changed" rows);
//  * int8 weights (per output row) with an optional SmoothQuant column scale
//    (same card, "Quantized" row and "How it was made");
//  * int4 weights with the per-row clip search ("MossInt4", "Format").
//
// Data layout and work split.  A row of K bf16 values is cut into virtual
// 256-element groups; four consecutive lanes own one group, 64 elements each.
// Lane L loads the 16-byte pieces 4i + L (i = 0..7) of its group, so the four
// lanes of a group read 64 contiguous bytes per load instruction.  Register
// j = 8i + r then holds element 32i + 8L + r: element bits 0-2 and 5-7 sit in
// registers and bits 3-4 in the lane index.  The FWHT runs six butterfly
// stages inside registers, then twice swaps a lane bit with a register bit
// through one shuffle per register pair and runs the remaining two stages in
// registers.  Afterwards lane L holds elements 32L + (j & 31) + 128 (j >> 5):
// two runs of 32 contiguous codes, stored with 16-byte stores.
//
// The 1/16 normalisation of H and the RMSNorm factor r are per-row scalars;
// they do not change the codes (codes depend on v / max|v| only), so they are
// folded into the fp64 computation of the per-row scale.
#pragma once

#include "ptx.cuh"

namespace convrot {

enum PreOp { PRE_NONE = 0, PRE_NORM = 1, PRE_COLSCALE = 2 };
// QK_BF16: no quantisation; the rotated (and normalised) row is stored in
// bf16 for the weight-only path
enum QuantKind { QK_INT8 = 0, QK_INT4 = 1, QK_BF16 = 2 };

struct RowQuantArgs {
  const uint16_t* src;  // [rows, K] bf16 bits
  const float* vec;     // [K]: RMSNorm weight w (PRE_NORM) or column scale (PRE_COLSCALE)
  int8_t* dst8;         // [rows, K]      (QK_INT8)
  uint8_t* dst4;        // [rows, K / 2]  (QK_INT4)
  uint16_t* dstb;       // [rows, K] bf16 (QK_BF16)
  float* scale;         // [rows]
  int rows;
  int K;
  float eps;
  float clip_lo;
  float clip_step;
  int clip_steps;
  int team;          // threads per row: 4, 8, 16, 32, or a multiple of 32 up to 256
  int rows_per_cta;  // rows handled by one CTA at a time (blockDim = team * rows_per_cta)
  int passes;        // chunks per thread (1 = row stays in registers)
};

constexpr int RQ_MAX_WARPS_PER_TEAM = 8;
constexpr int RQ_MAX_SLOTS = 8;

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// Reductions over the threads of one row team.  Teams of <= 32 threads are
// aligned power-of-two lane ranges inside a warp and reduce with shuffles;
// larger teams are whole warps and meet at a named barrier (one id per row
// slot).  Shared buffers alternate between two halves so that one barrier per
// reduction suffices.
struct TeamReducer {
  float* smax;   // [2][RQ_MAX_SLOTS][RQ_MAX_WARPS_PER_TEAM]
  double* ssum;  // [2][RQ_MAX_SLOTS][RQ_MAX_WARPS_PER_TEAM]
  int team, slot, lane, warp_in_team, nwarps;
  int parity;

  __device__ __forceinline__ void reduce(float& mx, double& sm) {
    const int width = team < 32 ? team : 32;
    for (int o = width >> 1; o > 0; o >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      sm += __shfl_xor_sync(0xffffffffu, sm, o);
    }
    if (team <= 32) return;
    const int base = (parity * RQ_MAX_SLOTS + slot) * RQ_MAX_WARPS_PER_TEAM;
    if (lane == 0) {
      smax[base + warp_in_team] = mx;
      ssum[base + warp_in_team] = sm;
    }
    named_bar_sync(1 + slot, team);
    mx = smax[base];
    sm = ssum[base];
    for (int w = 1; w < nwarps; ++w) {  // fixed order: deterministic sum
      mx = fmaxf(mx, smax[base + w]);
      sm += ssum[base + w];
    }
    parity ^= 1;
  }
};

// Loads the 64 elements lane L owns in virtual group g of one row and applies
// the per-column pre-operation.  Also accumulates sum(x^2) of the raw inputs
// (fp32 pairwise inside the thread).
template <int PRE>
__device__ __forceinline__ void rq_load(const RowQuantArgs& a, const uint16_t* row, int g, int L,
                                        bool ok, float (&v)[64], float& sq) {
  float part[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = g * 256 + i * 32 + L * 8;
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (ok && e < a.K) raw = ld_nc_v4(row + e);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      v[8 * i + 2 * h] = __uint_as_float(w[h] << 16);
      v[8 * i + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
    }
    float p0 = v[8 * i] * v[8 * i] + v[8 * i + 1] * v[8 * i + 1];
    float p1 = v[8 * i + 2] * v[8 * i + 2] + v[8 * i + 3] * v[8 * i + 3];
    float p2 = v[8 * i + 4] * v[8 * i + 4] + v[8 * i + 5] * v[8 * i + 5];
    float p3 = v[8 * i + 6] * v[8 * i + 6] + v[8 * i + 7] * v[8 * i + 7];
    part[i] = (p0 + p1) + (p2 + p3);
    if (PRE != PRE_NONE) {
      float4 m0 = make_float4(0.f, 0.f, 0.f, 0.f), m1 = m0;
      if (ok && e < a.K) {
        m0 = __ldg(reinterpret_cast<const float4*>(a.vec + e));
        m1 = __ldg(reinterpret_cast<const float4*>(a.vec + e + 4));
      }
      const float mm[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float mult = PRE == PRE_NORM ? 1.0f + mm[r] : mm[r];
        v[8 * i + r] *= mult;
      }
    }
  }
  sq += ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
}

// fp64 sum of squares of the raw inputs lane L owns in virtual group g (the
// rare path for rows whose fp32 sum of squares leaves the safe range).
__device__ __forceinline__ double rq_sumsq64(const RowQuantArgs& a, const uint16_t* row, int g,
                                             int L, bool ok) {
  double acc = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = g * 256 + i * 32 + L * 8;
    if (ok && e < a.K) {
      const uint4 raw = ld_nc_v4(row + e);
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

__device__ __forceinline__ void butterfly(float (&v)[64], int h) {
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    if (!(j & h)) {
      const float x = v[j], y = v[j + h];
      v[j] = x + y;
      v[j + h] = x - y;
    }
  }
}

// Exchanges register bit h with the lane bit m: afterwards register bit h
// indexes what the lane bit indexed before and vice versa.
__device__ __forceinline__ void lane_swap(float (&v)[64], int h, int m, int lane) {
  const bool upper = (lane & m) != 0;
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    if (!(j & h)) {
      const float send = upper ? v[j] : v[j + h];
      const float recv = __shfl_xor_sync(0xffffffffu, send, m);
      if (upper)
        v[j] = recv;
      else
        v[j + h] = recv;
    }
  }
}

// Unnormalised Walsh-Hadamard transform (natural Sylvester order) of the
// GRP-element groups within the 256 elements held by four lanes: GRP = 256
// runs all eight butterfly stages, GRP = 16 the stages of element bits 0-3,
// GRP = 0 only the data movement.
template <int GRP>
__device__ __forceinline__ void rq_transform(float (&v)[64], int lane) {
  static_assert(GRP == 0 || GRP == 16 || GRP == 256, "group size 0, 16 or 256");
  if (GRP) {
    butterfly(v, 1);   // element bit 0
    butterfly(v, 2);   // element bit 1
    butterfly(v, 4);   // element bit 2
  }
  if (GRP == 256) {
    butterfly(v, 8);   // element bit 5
    butterfly(v, 16);  // element bit 6
    butterfly(v, 32);  // element bit 7
  }
  lane_swap(v, 8, 1, lane);  // register bit 3 <-> element bit 3
  if (GRP) butterfly(v, 8);
  lane_swap(v, 16, 2, lane);  // register bit 4 <-> element bit 4
  if (GRP == 256) butterfly(v, 16);
}

// 1 / sqrt(GRP): the normalisation of H_GRP, applied to the per-row scale.
template <int GRP>
__host__ __device__ constexpr double group_norm() {
  return GRP == 256 ? 1.0 / 16.0 : (GRP == 16 ? 1.0 / 4.0 : 1.0);
}

__device__ __forceinline__ float rq_absmax(const float (&v)[64]) {
  float m0 = 0.f, m1 = 0.f, m2 = 0.f, m3 = 0.f;
#pragma unroll
  for (int j = 0; j < 64; j += 4) {
    m0 = fmaxf(m0, fabsf(v[j]));
    m1 = fmaxf(m1, fabsf(v[j + 1]));
    m2 = fmaxf(m2, fabsf(v[j + 2]));
    m3 = fmaxf(m3, fabsf(v[j + 3]));
  }
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

__device__ __forceinline__ int clamp_code(int q, int qmax) { return max(-qmax, min(qmax, q)); }

__device__ __forceinline__ void rq_store_int8(const RowQuantArgs& a, int8_t* row, int g, int L,
                                              bool ok, const float (&v)[64], float inv) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int j = 32 * h + 16 * q + 4 * k + b;
          const int c = clamp_code(__float2int_rn(v[j] * inv), 127);
          word |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * b);
        }
        w[k] = word;
      }
      const int e = g * 256 + 128 * h + 32 * L + 16 * q;
      if (ok && e < a.K) st_v4(row + e, make_uint4(w[0], w[1], w[2], w[3]));
    }
  }
}

// The rotated values times `scale`, rounded once to bf16 (register j of the
// 32h + 16q block holds element g*256 + 128h + 32L + 16q + (j mod 16)).
__device__ __forceinline__ void rq_store_bf16(const RowQuantArgs& a, uint16_t* row, int g, int L,
                                              bool ok, const float (&v)[64], float scale) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t w[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int j = 32 * h + 16 * q + 2 * k;
        const __nv_bfloat162 b = __floats2bfloat162_rn(v[j] * scale, v[j + 1] * scale);
        w[k] = *reinterpret_cast<const uint32_t*>(&b);
      }
      const int e = g * 256 + 128 * h + 32 * L + 16 * q;
      if (ok && e < a.K) {
        st_v4(row + e, make_uint4(w[0], w[1], w[2], w[3]));
        st_v4(row + e + 8, make_uint4(w[4], w[5], w[6], w[7]));
      }
    }
  }
}

__device__ __forceinline__ float rq_sse_int4(const float (&v)[64], float s) {
  float e0 = 0.f, e1 = 0.f;
#pragma unroll
  for (int j = 0; j < 64; j += 2) {
    const float q0 = static_cast<float>(clamp_code(__float2int_rn(__fdiv_rn(v[j], s)), 7));
    const float q1 = static_cast<float>(clamp_code(__float2int_rn(__fdiv_rn(v[j + 1], s)), 7));
    const float d0 = v[j] - s * q0;
    const float d1 = v[j + 1] - s * q1;
    e0 = fmaf(d0, d0, e0);
    e1 = fmaf(d1, d1, e1);
  }
  return e0 + e1;
}

__device__ __forceinline__ void rq_store_int4(const RowQuantArgs& a, uint8_t* row, int g, int L,
                                              bool ok, const float (&v)[64], float s) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t word = 0;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const int j = 32 * h + 8 * k + b;
        const int c = s > 0.f ? clamp_code(__float2int_rn(__fdiv_rn(v[j], s)), 7) : 0;
        word |= (static_cast<uint32_t>(c) & 0xFu) << (4 * b);
      }
      w[k] = word;
    }
    const int e = g * 256 + 128 * h + 32 * L;  // first element of the run
    if (ok && e < a.K) st_v4(row + e / 2, make_uint4(w[0], w[1], w[2], w[3]));
  }
}

template <int GRP, int PRE, int QK, bool RESIDENT>
__global__ void __launch_bounds__(256) rowquant_kernel(RowQuantArgs a) {
  __shared__ float s_max[2 * RQ_MAX_SLOTS * RQ_MAX_WARPS_PER_TEAM];
  __shared__ double s_sum[2 * RQ_MAX_SLOTS * RQ_MAX_WARPS_PER_TEAM];
  pdl_launch_dependents();  // the grid is co-resident: dependents only take idle SMs
  pdl_wait();

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int slot = tid / a.team;
  const int t = tid - slot * a.team;
  const int L = t & 3;
  const int G = (a.K + 255) >> 8;  // virtual 256-groups per row

  TeamReducer red{s_max, s_sum, a.team, slot, lane, t >> 5, a.team >> 5, 0};

  const int row_blocks = (a.rows + a.rows_per_cta - 1) / a.rows_per_cta;
  for (int rb = blockIdx.x; rb < row_blocks; rb += gridDim.x) {
    const int row = rb * a.rows_per_cta + slot;
    const bool row_ok = row < a.rows;
    const uint16_t* src_row = a.src + static_cast<size_t>(row_ok ? row : 0) * a.K;

    float v[64];
    float sq = 0.f;
    float amax = 0.f;
    if (RESIDENT) {
      const int g = t >> 2;
      rq_load<PRE>(a, src_row, g, L, row_ok && g < G, v, sq);
      rq_transform<GRP>(v, lane);
      amax = rq_absmax(v);
    } else {
      for (int p = 0; p < a.passes; ++p) {
        const int g = (t + p * a.team) >> 2;
        rq_load<PRE>(a, src_row, g, L, row_ok && g < G, v, sq);
        rq_transform<GRP>(v, lane);
        amax = fmaxf(amax, rq_absmax(v));
      }
    }
    double sumsq = static_cast<double>(sq);
    red.reduce(amax, sumsq);
    if (PRE == PRE_NORM) {
      // The fp32 squares overflow for |x| above ~1e18 and underflow for rows of
      // tiny values; such rows (never seen in practice) get an fp64 recompute.
      // The decision is made warp-wide so that every shuffle stays converged.
      const bool need = amax > 0.f && !(sumsq > 0x1p-100 && sumsq < 0x1p+100);
      if (__any_sync(0xffffffffu, need)) {
        double s64 = 0.0;
        for (int p = 0; p < a.passes; ++p) {
          const int g = (t + p * a.team) >> 2;
          s64 += rq_sumsq64(a, src_row, g, L, row_ok && g < G);
        }
        float dummy = 0.f;
        red.reduce(dummy, s64);
        if (need) sumsq = s64;
      }
    }

    // fp64 per-row scale: absmax of the unnormalised transform, times
    // 1/sqrt(GRP) for the normalised Hadamard, times r for the RMSNorm.
    double rowfac = group_norm<GRP>();
    if (PRE == PRE_NORM) {
      const double ms = sumsq / static_cast<double>(a.K);
      rowfac *= 1.0 / sqrt(ms + static_cast<double>(a.eps));
    }

    if (QK == QK_BF16) {
      const float scale = static_cast<float>(rowfac);
      uint16_t* dst_row = a.dstb + static_cast<size_t>(row_ok ? row : 0) * a.K;
      if (RESIDENT) {
        const int g = t >> 2;
        rq_store_bf16(a, dst_row, g, L, row_ok && g < G, v, scale);
      } else {
        for (int p = 0; p < a.passes; ++p) {
          const int g = (t + p * a.team) >> 2;
          float sq2 = 0.f;
          rq_load<PRE>(a, src_row, g, L, row_ok && g < G, v, sq2);
          rq_transform<GRP>(v, lane);
          rq_store_bf16(a, dst_row, g, L, row_ok && g < G, v, scale);
        }
      }
    } else if (QK == QK_INT8) {
      const float inv = amax > 0.f ? 127.0f / amax : 0.0f;
      if (row_ok && t == 0)
        a.scale[row] = amax > 0.f ? static_cast<float>(static_cast<double>(amax) * rowfac / 127.0) : 0.0f;
      int8_t* dst_row = a.dst8 + static_cast<size_t>(row_ok ? row : 0) * a.K;
      if (RESIDENT) {
        const int g = t >> 2;
        rq_store_int8(a, dst_row, g, L, row_ok && g < G, v, inv);
      } else {
        for (int p = 0; p < a.passes; ++p) {
          const int g = (t + p * a.team) >> 2;
          float sq2 = 0.f;
          rq_load<PRE>(a, src_row, g, L, row_ok && g < G, v, sq2);
          rq_transform<GRP>(v, lane);
          rq_store_int8(a, dst_row, g, L, row_ok && g < G, v, inv);
        }
      }
    } else {
      // clip search: s_c = c * amax / 7 on the unnormalised transform
      float best_err = 0.f, best_s = 0.f;
      for (int ci = 0; ci < a.clip_steps; ++ci) {
        const float c = a.clip_lo + a.clip_step * static_cast<float>(ci);
        const float s = __fdiv_rn(c * amax, 7.0f);
        float err = 0.f;
        if (s > 0.f) {
          if (RESIDENT) {
            err = rq_sse_int4(v, s);
          } else {
            for (int p = 0; p < a.passes; ++p) {
              const int g = (t + p * a.team) >> 2;
              float sq2 = 0.f;
              rq_load<PRE>(a, src_row, g, L, row_ok && g < G, v, sq2);
              rq_transform<GRP>(v, lane);
              err += rq_sse_int4(v, s);
            }
          }
        }
        float dummy = 0.f;
        double e64 = static_cast<double>(err);
        red.reduce(dummy, e64);
        const float e = static_cast<float>(e64);
        if (ci == 0 || e < best_err) {
          best_err = e;
          best_s = s;
        }
      }
      if (row_ok && t == 0)
        a.scale[row] = best_s > 0.f ? static_cast<float>(static_cast<double>(best_s) * rowfac) : 0.0f;
      uint8_t* dst_row = a.dst4 + static_cast<size_t>(row_ok ? row : 0) * (a.K / 2);
      if (RESIDENT) {
        const int g = t >> 2;
        rq_store_int4(a, dst_row, g, L, row_ok && g < G, v, best_s);
      } else {
        for (int p = 0; p < a.passes; ++p) {
          const int g = (t + p * a.team) >> 2;
          float sq2 = 0.f;
          rq_load<PRE>(a, src_row, g, L, row_ok && g < G, v, sq2);
          rq_transform<GRP>(v, lane);
          rq_store_int4(a, dst_row, g, L, row_ok && g < G, v, best_s);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// SmoothQuant calibration (offline): column maxima of the normalised
// activation and of the weight, then s = ax^alpha / aw^(1-alpha).
// ---------------------------------------------------------------------------
constexpr int CAL_ROWS = 64;

// ax[c] = max over rows of |x[m,c] * r_m * (1 + w[c])|, as float bits in an
// unsigned max (order-preserving for non-negative floats).  w == nullptr: the
// activation reaches the linear as it is (ax[c] = max |x[m,c]|).
__global__ void __launch_bounds__(256) calib_act_colmax(const uint16_t* x, int M, int K,
                                                        const float* w, float eps,
                                                        unsigned* axbits) {
  __shared__ float s_r[CAL_ROWS];
  const int m0 = blockIdx.x * CAL_ROWS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int rr = warp; rr < CAL_ROWS && w == nullptr; rr += 8)
    if (lane == 0) s_r[rr] = 1.0f;
  for (int rr = warp; rr < CAL_ROWS && w != nullptr; rr += 8) {
    const int m = m0 + rr;
    double acc = 0.0;
    if (m < M) {
      const uint16_t* row = x + static_cast<size_t>(m) * K;
      for (int k = lane; k < K; k += 32) {
        const double f = static_cast<double>(__uint_as_float(static_cast<uint32_t>(row[k]) << 16));
        acc += f * f;
      }
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) s_r[rr] = static_cast<float>(1.0 / sqrt(acc / K + static_cast<double>(eps)));
  }
  __syncthreads();
  for (int c = threadIdx.x; c < K; c += blockDim.x) {
    const float mult = w != nullptr ? 1.0f + w[c] : 1.0f;
    float mx = 0.f;
    for (int rr = 0; rr < CAL_ROWS && m0 + rr < M; ++rr) {
      const float xv = __uint_as_float(static_cast<uint32_t>(x[static_cast<size_t>(m0 + rr) * K + c]) << 16);
      mx = fmaxf(mx, fabsf(xv * s_r[rr] * mult));
    }
    atomicMax(axbits + c, __float_as_uint(mx));
  }
}

__global__ void __launch_bounds__(256) calib_weight_colmax(const uint16_t* W, int N, int K,
                                                           unsigned* awbits) {
  const int n0 = blockIdx.x * CAL_ROWS;
  for (int c = threadIdx.x; c < K; c += blockDim.x) {
    float mx = 0.f;
    for (int rr = 0; rr < CAL_ROWS && n0 + rr < N; ++rr) {
      mx = fmaxf(mx, fabsf(__uint_as_float(static_cast<uint32_t>(W[static_cast<size_t>(n0 + rr) * K + c]) << 16)));
    }
    atomicMax(awbits + c, __float_as_uint(mx));
  }
}

// In place: smooth holds ax bits, folded holds aw bits on entry.
__global__ void __launch_bounds__(256) calib_finalize(const float* w, int K, float alpha,
                                                      float* smooth, float* folded) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= K) return;
  const double ax = static_cast<double>(smooth[c]);
  const double aw = static_cast<double>(folded[c]);
  double s = 1.0;
  if (ax > 0.0 && aw > 0.0) s = pow(ax, static_cast<double>(alpha)) / pow(aw, 1.0 - alpha);
  s = fmin(fmax(s, 1e-5), 1e5);
  smooth[c] = static_cast<float>(s);
  if (w != nullptr) folded[c] = static_cast<float>((1.0 + static_cast<double>(w[c])) / s - 1.0);
}

// ---------------------------------------------------------------------------
// MLP boundary preparation (offline)
// ---------------------------------------------------------------------------
// Rows of gate and up in alternating blocks of SWIGLU_BLOCK: output row r is
// gate row 16 (r / 32) + r % 32 when r % 32 < 16, else the up row 16 (r / 32)
// + r % 32 - 16.  Rows are copied as 32-bit words.
__global__ void __launch_bounds__(256) interleave_rows_kernel(const uint32_t* g, const uint32_t* u,
                                                              uint32_t* out, size_t I, size_t wpr) {
  const size_t total = 2 * I * wpr;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t r = i / wpr, w = i - r * wpr;
    const size_t blk = r / 32, k = r % 32;
    const uint32_t* src = k < 16 ? g : u;
    out[i] = src[(16 * blk + (k & 15)) * wpr + w];
  }
}

// s_row[i] / smooth[i]: a per-channel scale 1 / smooth folded into the rows of
// a row-quantised weight (the codes of a row do not change when it is scaled)
__global__ void __launch_bounds__(256) fold_row_scales_kernel(float* s_row, const float* smooth,
                                                              int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) s_row[i] = s_row[i] / smooth[i];
}

}  // namespace convrot
