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
// Activation rotate-quantise for the per-token hot path, fed by TMA.
//
// One CTA per SM.  Warp 0 (one lane) streams "stages" of R consecutive token
// rows into a ring of shared-memory buffers with 1-D bulk copies (one copy per
// stage: the rows are contiguous in HBM) and prefetches later stages into L2.
// The other warps form R teams of T = (padded) K/64 threads; team r takes row r
// of a stage, reads its 64 elements per thread from shared memory in the same
// lane layout as rowquant_kernel, releases the stage at once, and runs the
// 256-point FWHT in packed f32x2 arithmetic (lane bits by shuffles), the row
// reductions and 8-byte code stores.  The RMSNorm weight w is bulk-copied once
// per CTA into shared memory together with the first rows.
// ---------------------------------------------------------------------------
constexpr int ACT_MAX_STAGES = 8;

struct ActArgs {
  const uint16_t* x;   // [M, K] bf16 bits
  const float* norm_w; // [K] or null
  int8_t* xq;          // [M, K]
  float* s_tok;        // [M]
  int M, K;
  float eps;
  int team;            // threads per row (as rowquant_kernel)
  int rows;            // rows per stage (teams per CTA)
  int stages;
  int wsm_bytes;       // shared bytes for 1 + w (K * 4 rounded up to 1024, or 0)
};

__device__ __forceinline__ uint32_t q8_byte(float v, float inv) {
  // rint(v * inv) in one rounding: adding 1.5 * 2^23 leaves the integer in the
  // low mantissa bits (round-half-even); its low byte is the two's-complement
  // int8 code (|v * inv| <= 127 by construction of inv)
  return __float_as_uint(fmaf(v, inv, 12582912.0f));
}

__device__ __forceinline__ uint32_t pack4_bytes(uint32_t q0, uint32_t q1, uint32_t q2, uint32_t q3) {
  return __byte_perm(__byte_perm(q0, q1, 0x0040), __byte_perm(q2, q3, 0x0040), 0x5410);
}

__device__ __forceinline__ void act_store_int8(int8_t* row, int K, int g, int L, bool ok,
                                               const float (&v)[64], float inv) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int j = 32 * h + 16 * q + 4 * k;
        w[k] = pack4_bytes(q8_byte(v[j], inv), q8_byte(v[j + 1], inv), q8_byte(v[j + 2], inv),
                           q8_byte(v[j + 3], inv));
      }
      const int e = g * 256 + 128 * h + 32 * L + 16 * q;
      if (ok && e < K) st_v4(row + e, make_uint4(w[0], w[1], w[2], w[3]));
    }
  }
}

template <bool NORM>
__device__ __forceinline__ void act_load_smem(const uint16_t* srow, const float* wsm, int K, int g,
                                              int L, bool ok, float (&v)[64], float& sq) {
  float part[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = g * 256 + i * 32 + L * 8;
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (ok && e < K) raw = *reinterpret_cast<const uint4*>(srow + e);
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
    if (NORM) {
      float4 m0 = make_float4(0.f, 0.f, 0.f, 0.f), m1 = m0;
      if (ok && e < K) {
        m0 = *reinterpret_cast<const float4*>(wsm + e);
        m1 = *reinterpret_cast<const float4*>(wsm + e + 4);
      }
      v[8 * i] *= m0.x; v[8 * i + 1] *= m0.y; v[8 * i + 2] *= m0.z; v[8 * i + 3] *= m0.w;
      v[8 * i + 4] *= m1.x; v[8 * i + 5] *= m1.y; v[8 * i + 6] *= m1.z; v[8 * i + 7] *= m1.w;
    }
  }
  sq += ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
}

// Packed fp32x2 arithmetic (one instruction for two lanes of a 64-bit register).
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
  return static_cast<uint64_t>(__float_as_uint(lo)) | (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }

// Lane (g, L) of a 256-group holds elements 32i + 8L + r (i, r = 0..7) as 32
// pairs: pair p = 4i + r/2 holds (r even, r odd).  Loads them from a staged
// row in shared memory, accumulates sum(x^2) and applies the norm multiplier
// 1 + w (wsm holds w).
// WHOLE: K is a multiple of 256, so a lane whose group exists is in range.
template <bool NORM, bool WHOLE>
__device__ __forceinline__ void act3_load(const uint16_t* srow, const float* wsm, int K, int g,
                                          int L, bool ok, uint64_t (&v)[32], float& sq) {
  float part[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = g * 256 + i * 32 + L * 8;
    const bool in = WHOLE ? ok : (ok && e < K);
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (in) raw = ld_shared_v4(srow + e);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint64_t acc = 0;
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const uint64_t x2 = static_cast<uint64_t>(w[h] << 16) | (static_cast<uint64_t>(w[h] & 0xFFFF0000u) << 32);
      acc = h == 0 ? f2_mul(x2, x2) : f2_fma(x2, x2, acc);
      v[4 * i + h] = x2;
    }
    part[i] = f2_lo(acc) + f2_hi(acc);
    if (NORM) {
      ulonglong2 m0 = make_ulonglong2(0ull, 0ull), m1 = m0;
      if (in) {
        const uint4 u0 = ld_shared_v4(wsm + e), u1 = ld_shared_v4(wsm + e + 4);
        m0 = make_ulonglong2(u0.x | (static_cast<uint64_t>(u0.y) << 32),
                             u0.z | (static_cast<uint64_t>(u0.w) << 32));
        m1 = make_ulonglong2(u1.x | (static_cast<uint64_t>(u1.y) << 32),
                             u1.z | (static_cast<uint64_t>(u1.w) << 32));
      }
      // x * (1 + w) as x + x * w: one rounding of the exact product
      v[4 * i] = f2_fma(v[4 * i], m0.x, v[4 * i]);
      v[4 * i + 1] = f2_fma(v[4 * i + 1], m0.y, v[4 * i + 1]);
      v[4 * i + 2] = f2_fma(v[4 * i + 2], m1.x, v[4 * i + 2]);
      v[4 * i + 3] = f2_fma(v[4 * i + 3], m1.y, v[4 * i + 3]);
    }
  }
  sq += ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
}

// Unnormalised FWHT of the GRP-element groups (256 or 16) within the 256
// elements held by four lanes, in place.
template <int GRP>
__device__ __forceinline__ void act3_fwht(uint64_t (&v)[32], int lane) {
  // element bit 0: inside each pair
#pragma unroll
  for (int p = 0; p < 32; ++p) {
    const float x = f2_lo(v[p]), y = f2_hi(v[p]);
    v[p] = f2_pack(x + y, x - y);
  }
  // element bits 1, 2 (and 5, 6, 7 for 256-point groups): between pairs
  // (pair-index bits 0..4)
#pragma unroll
  for (int m = 1; m < (GRP == 256 ? 32 : 4); m <<= 1) {
#pragma unroll
    for (int p = 0; p < 32; ++p) {
      if (!(p & m)) {
        const uint64_t x = v[p], y = v[p | m];
        v[p] = f2_add(x, y);
        v[p | m] = f2_sub(x, y);
      }
    }
  }
  // element bits 3 (and 4): between lanes (lane bits 0, 1).  The lane whose
  // bit is clear keeps x + partner, the other partner - x.
#pragma unroll
  for (int lm = 1; lm <= (GRP == 256 ? 2 : 1); lm <<= 1) {
    const float sg = (lane & lm) ? -1.0f : 1.0f;
    const uint64_t s2 = f2_pack(sg, sg);
#pragma unroll
    for (int p = 0; p < 32; ++p) {
      const uint32_t lo = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v[p]), lm);
      const uint32_t hi = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v[p] >> 32), lm);
      v[p] = f2_fma(v[p], s2, static_cast<uint64_t>(lo) | (static_cast<uint64_t>(hi) << 32));
    }
  }
}

__device__ __forceinline__ float act3_absmax(const uint64_t (&v)[32]) {
  float m0 = 0.f, m1 = 0.f, m2 = 0.f, m3 = 0.f;
#pragma unroll
  for (int p = 0; p < 32; p += 2) {
    m0 = fmaxf(m0, fabsf(f2_lo(v[p])));
    m1 = fmaxf(m1, fabsf(f2_hi(v[p])));
    m2 = fmaxf(m2, fabsf(f2_lo(v[p + 1])));
    m3 = fmaxf(m3, fabsf(f2_hi(v[p + 1])));
  }
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

// int8 codes rint(v * inv) (one rounding, half-even), 8 bytes per i.
template <bool WHOLE>
__device__ __forceinline__ void act3_store(int8_t* row, int K, int g, int L, bool ok,
                                           const uint64_t (&v)[32], float inv) {
  const uint64_t inv2 = f2_pack(inv, inv);
  const uint64_t mag2 = f2_pack(12582912.0f, 12582912.0f);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t q[8];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const uint64_t t = f2_fma(v[4 * i + h], inv2, mag2);
      q[2 * h] = static_cast<uint32_t>(t);
      q[2 * h + 1] = static_cast<uint32_t>(t >> 32);
    }
    const uint32_t w0 = pack4_bytes(q[0], q[1], q[2], q[3]);
    const uint32_t w1 = pack4_bytes(q[4], q[5], q[6], q[7]);
    const int e = g * 256 + i * 32 + L * 8;
    if (WHOLE ? ok : (ok && e < K))
      asm volatile("st.global.v2.u32 [%0], {%1, %2};" ::"l"(row + e), "r"(w0), "r"(w1) : "memory");
  }
}

template <int GRP, bool NORM>
__global__ void __launch_bounds__(416, 1) actquant_kernel(ActArgs a) {
  // K is a multiple of 256 for 256-point groups: no per-element bounds checks
  constexpr bool WHOLE = GRP == 256;
  pdl_launch_dependents();  // the grid is co-resident: dependents only take idle SMs
  __shared__ float s_max[2 * RQ_MAX_SLOTS * RQ_MAX_WARPS_PER_TEAM];
  __shared__ double s_sum[2 * RQ_MAX_SLOTS * RQ_MAX_WARPS_PER_TEAM];
  __shared__ uint64_t full[ACT_MAX_STAGES], empty[ACT_MAX_STAGES], wbar;
  __shared__ int abort_word;
  extern __shared__ __align__(1024) uint8_t act_smem[];
  float* wsm = reinterpret_cast<float*>(act_smem);
  uint8_t* ring = act_smem + a.wsm_bytes;
  const int stage_bytes = a.rows * a.K * 2;
  volatile int* abort_flag = &abort_word;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int consumers = a.team * a.rows;
  const int cwarps = consumers >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], cwarps);
    }
    mbar_init(&wbar, 1);
    abort_word = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();  // x, w, Xq and s_tok may belong to the previous kernel

  const int units = (a.M + a.rows - 1) / a.rows;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      if (NORM) {
        // the norm weight w [K] fp32, copied once per CTA next to the first rows
        mbar_arrive_expect_tx(&wbar, static_cast<uint32_t>(a.K) * 4u);
        bulk_load_1d(wsm, a.norm_w, static_cast<uint32_t>(a.K) * 4u, &wbar);
      }
      int i = 0;
      for (int u = blockIdx.x; u < units; u += gridDim.x, ++i) {
        const int s = i % a.stages;
        const uint32_t ph = (i / a.stages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, SITE_PROD_EMPTY)) break;
        const int r0 = u * a.rows;
        const int nrows = min(a.rows, a.M - r0);
        const uint32_t bytes = static_cast<uint32_t>(nrows) * a.K * 2;
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_load_1d(ring + s * stage_bytes, a.x + static_cast<size_t>(r0) * a.K, bytes, &full[s]);
        // warm L2 with the unit this CTA loads `stages` steps later
        const int uf = u + a.stages * gridDim.x;
        if (uf < units) {
          const int rf = uf * a.rows;
          bulk_prefetch_l2(a.x + static_cast<size_t>(rf) * a.K,
                           static_cast<uint32_t>(min(a.rows, a.M - rf)) * a.K * 2);
        }
      }
      // drain: every issued copy has landed (consumers waited on each) unless
      // a wait gave up; wait (bounded) for the last ones before exiting
      const int issued = i;
      for (int j = max(0, issued - a.stages); j < issued; ++j) {
        int dummy = 0;
        mbar_wait(&full[j % a.stages], (j / a.stages) & 1u, &dummy, SITE_DRAIN);
      }
      if (NORM) {
        int dummy = 0;
        mbar_wait(&wbar, 0u, &dummy, SITE_DRAIN);
      }
    }
    return;
  }
  // ------------------------------------------------------------ consumers
  const int ct = threadIdx.x - 32;
  const int slot = ct / a.team;
  const int t = ct - slot * a.team;
  const int L = t & 3;
  const int g = t >> 2;
  const int G = (a.K + 255) >> 8;
  TeamReducer red{s_max, s_sum, a.team, slot, lane, t >> 5, a.team >> 5, 0};
  if (NORM && !mbar_wait(&wbar, 0u, abort_flag, SITE_EPI_FULL)) return;
  int i = 0;
  for (int u = blockIdx.x; u < units; u += gridDim.x, ++i) {
    const int s = i % a.stages;
    const uint32_t ph = (i / a.stages) & 1u;
    const bool got = mbar_wait(&full[s], ph, abort_flag, SITE_EPI_FULL);
    // every consumer warp takes the same decision (abort is CTA-wide), so the
    // team reductions below stay matched
    if (!got) break;
    const int row = u * a.rows + slot;
    const bool row_ok = row < a.M;
    const uint16_t* srow =
        reinterpret_cast<const uint16_t*>(ring + s * stage_bytes) + static_cast<size_t>(slot) * a.K;
    uint64_t v[32];
    float sq = 0.f;
    act3_load<NORM, WHOLE>(srow, wsm, a.K, g, L, row_ok && g < G, v, sq);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);  // stage read: the producer may refill it
    if (GRP) act3_fwht<GRP>(v, lane);
    float amax = act3_absmax(v);
    double sumsq = static_cast<double>(sq);
    red.reduce(amax, sumsq);
    if (NORM) {
      const bool need = amax > 0.f && !(sumsq > 0x1p-100 && sumsq < 0x1p+100);
      if (__any_sync(0xffffffffu, need)) {
        const uint16_t* grow = a.x + static_cast<size_t>(row_ok ? row : 0) * a.K;
        RowQuantArgs ra{};
        ra.K = a.K;
        double s64 = rq_sumsq64(ra, grow, g, L, row_ok && g < G);
        float dummy = 0.f;
        red.reduce(dummy, s64);
        if (need) sumsq = s64;
      }
    }
    const float inv = amax > 0.f ? 127.0f / amax : 0.0f;
    if (row_ok && t == 0) {
      // the per-row scale is needed by one thread only
      double rowfac = group_norm<GRP>();
      if (NORM) rowfac *= 1.0 / sqrt(sumsq / static_cast<double>(a.K) + static_cast<double>(a.eps));
      a.s_tok[row] = amax > 0.f ? static_cast<float>(static_cast<double>(amax) * rowfac / 127.0) : 0.0f;
    }
    act3_store<WHOLE>(a.xq + static_cast<size_t>(row_ok ? row : 0) * a.K, a.K, g, L, row_ok && g < G,
                    v, inv);
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
