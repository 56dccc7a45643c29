// Parameters of the grouped AWQ projection kernels (both tile paths).
#pragma once

#include "common.cuh"

namespace moe {

struct ProjParams {
  const uint16_t *x;  // [A, K] activations, or [T, K] read through `gather`
  const int32_t *gather;  // NULL, or [A]: batch row r is x row gather[r] (in [0, T))
  int64_t T;              // rows of x when gathering
  int act_dt;
  int64_t A, K, N;
  const int32_t *offsets;
  int E;
  const int32_t *qw[2];
  const int32_t *qz[2];
  const uint16_t *sc[2];
  const void *bias[2];
  int bias_dt;
  int group;
  uint16_t *out;   // [A, N]: h (two projections) or y (one)
  uint16_t *gout;  // G (two projections), or NULL
  uint16_t *uout;  // U (two projections), or NULL
  int32_t *status;
  // split-K scratch of the streaming tile (workspace)
  float *partials;
  int32_t *counters;
  int kq;  // K splits
  int preconv;  // x holds F16 copies of BF16 activations
  int odt;      // dtype of gout and uout, and of out with one projection (F16 or BF16)
  int hdt;      // dtype of out (h) with two projections
#ifdef MOE_TEST_HOOKS
  int test_stall;  // test build only: see moe_test_arm_stall
#endif
};

struct BwdParams {
  const uint16_t *grad[2];  // [A, N] each
  int gdt;
  int64_t A, N, K;
  const int32_t *offsets;
  int E;
  const int32_t *qw[2];
  const int32_t *qz[2];
  const uint16_t *sc[2];
  int group;
  uint16_t *out;  // [A, K]
  int32_t *status;
  int preconv;  // grad holds F16 copies of BF16 gradients
  int odt;      // dtype of out (F16 or BF16), independent of the gradients'
};

// Row of x that batch row r reads: r itself, or gather[r] (an index outside
// [0, T) is reported and row 0 is read instead).
__device__ __forceinline__ int64_t act_row(const ProjParams &p, int64_t r) {
  if (!p.gather) return r;
  const int32_t v = __ldg(p.gather + r);
  if (v < 0 || (int64_t)v >= p.T) {
    report(p.status, MOE_DEVICE_ERR_ROW_RANGE);
    return 0;
  }
  return v;
}

// 8 bias values n0.. of local expert e (0 without a bias), with 16-byte loads.
__device__ __forceinline__ void bias8(const void *bias, int dt, int64_t i0, float (&b)[8]) {
  if (!bias) {
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = 0.f;
  } else if (dt == MOE_F32) {
    const float4 *q = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(bias) + i0);
    const float4 v0 = __ldg(q), v1 = __ldg(q + 1);
    b[0] = v0.x, b[1] = v0.y, b[2] = v0.z, b[3] = v0.w, b[4] = v1.x, b[5] = v1.y, b[6] = v1.z, b[7] = v1.w;
  } else {
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(bias) + i0));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      b[2 * i] = bits_to_f32((uint16_t)(w[i] & 0xFFFFu), dt);
      b[2 * i + 1] = bits_to_f32((uint16_t)(w[i] >> 16), dt);
    }
  }
}

// Two FP32 values rounded (RNE) to the activation dtype, packed low/high.
template <bool BF>
__device__ __forceinline__ uint32_t round_pair(float a, float b) {
  if (BF) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&v);
  }
  const __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t *>(&v);
}

template <bool BF>
__device__ __forceinline__ float2 unpack_pair(uint32_t v) {
  return make_float2(bits_to_f32((uint16_t)(v & 0xFFFFu), BF ? MOE_BF16 : MOE_F16),
                     bits_to_f32((uint16_t)(v >> 16), BF ? MOE_BF16 : MOE_F16));
}

// silu(G) U from the rounded G and U.  Fast exponential and division: their
// few-ulp FP32 error is far below one rounding of the 16-bit result.
__device__ __forceinline__ float swiglu1(float G, float U) { return __fdividef(G, 1.f + __expf(-G)) * U; }

// Two h values rounded to p.hdt.  F16 h from BF16 G and U (gu_bf): a value
// that is not +-inf but becomes inf or NaN in F16 is reported as
// MOE_DEVICE_ERR_ACT_RANGE, the rule of the BF16 -> F16 input conversion.
__device__ __forceinline__ uint32_t round_h(const ProjParams &p, float a, float b, bool gu_bf) {
  if (p.hdt == MOE_BF16) return round_pair<true>(a, b);
  const uint32_t r = round_pair<false>(a, b);
  if (gu_bf && ((((r & 0x7C00u) == 0x7C00u) && !isinf(a)) || (((r & 0x7C000000u) == 0x7C000000u) && !isinf(b))))
    report(p.status, MOE_DEVICE_ERR_ACT_RANGE);
  return r;
}

template <int NPROJ, bool BF>
__device__ __forceinline__ void finish8_t(const ProjParams &p, int e, int64_t row, int64_t n0, const float *g,
                                          const float *u) {
  float bg[8];
  bias8(p.bias[0], p.bias_dt, (int64_t)e * p.N + n0, bg);
  uint32_t o[4];
  if (NPROJ == 2) {
    float bu[8];
    bias8(p.bias[1], p.bias_dt, (int64_t)e * p.N + n0, bu);
    uint32_t og[4], ou[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      og[i] = round_pair<BF>(g[2 * i] + bg[2 * i], g[2 * i + 1] + bg[2 * i + 1]);
      ou[i] = round_pair<BF>(u[2 * i] + bu[2 * i], u[2 * i + 1] + bu[2 * i + 1]);
      const float2 G = unpack_pair<BF>(og[i]), U = unpack_pair<BF>(ou[i]);
      o[i] = round_h(p, swiglu1(G.x, U.x), swiglu1(G.y, U.y), BF);
    }
    if (p.gout) *reinterpret_cast<uint4 *>(p.gout + row * p.N + n0) = make_uint4(og[0], og[1], og[2], og[3]);
    if (p.uout) *reinterpret_cast<uint4 *>(p.uout + row * p.N + n0) = make_uint4(ou[0], ou[1], ou[2], ou[3]);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = round_pair<BF>(g[2 * i] + bg[2 * i], g[2 * i + 1] + bg[2 * i + 1]);
  }
  *reinterpret_cast<uint4 *>(p.out + row * p.N + n0) = make_uint4(o[0], o[1], o[2], o[3]);
}

// finish8_t with the bias of the 8 columns already in registers (bg, bu).
template <int NPROJ, bool BF>
__device__ __forceinline__ void finish8_bt(const ProjParams &p, int64_t row, int64_t n0, const float *g, const float *u,
                                           const float *bg, const float *bu) {
  uint32_t o[4];
  if (NPROJ == 2) {
    uint32_t og[4], ou[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      og[i] = round_pair<BF>(g[2 * i] + bg[2 * i], g[2 * i + 1] + bg[2 * i + 1]);
      ou[i] = round_pair<BF>(u[2 * i] + bu[2 * i], u[2 * i + 1] + bu[2 * i + 1]);
      const float2 G = unpack_pair<BF>(og[i]), U = unpack_pair<BF>(ou[i]);
      o[i] = round_h(p, swiglu1(G.x, U.x), swiglu1(G.y, U.y), BF);
    }
    if (p.gout) *reinterpret_cast<uint4 *>(p.gout + row * p.N + n0) = make_uint4(og[0], og[1], og[2], og[3]);
    if (p.uout) *reinterpret_cast<uint4 *>(p.uout + row * p.N + n0) = make_uint4(ou[0], ou[1], ou[2], ou[3]);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = round_pair<BF>(g[2 * i] + bg[2 * i], g[2 * i + 1] + bg[2 * i + 1]);
  }
  *reinterpret_cast<uint4 *>(p.out + row * p.N + n0) = make_uint4(o[0], o[1], o[2], o[3]);
}

// Final values of 8 consecutive output columns n0.. of row `row` of local
// expert e from FP32 sums (gate sums g, up sums u for the pair): bias, one
// rounding to the output dtype, SwiGLU from the rounded G and U.
template <int NPROJ>
__device__ __forceinline__ void finish8(const ProjParams &p, int e, int64_t row, int64_t n0, const float *g,
                                        const float *u) {
  if (p.odt == MOE_BF16) finish8_t<NPROJ, true>(p, e, row, n0, g, u);
  else finish8_t<NPROJ, false>(p, e, row, n0, g, u);
}

void launch_fwd_mma(const ProjParams &p, int nproj, bool bf16_mma, int nt, cudaStream_t st);
void launch_bwd_mma(const BwdParams &p, int nproj, bool bf16_mma, int nt, cudaStream_t st);
void launch_dump(const int32_t *qw, const int32_t *qz, const uint16_t *sc, int64_t K, int64_t N, int group,
                 uint16_t *out, int mode, bool bf16_mma, cudaStream_t st);
struct StreamPlan {
  bool fits;      // the streaming tile can run this shape
  int rows;       // input rows per pipeline stage (32 or 64)
  int kq;         // K splits across CTAs
  size_t bytes;   // workspace bytes (partials + counters)
  size_t partial_off, counter_off;
};
StreamPlan stream_plan(int64_t A, int64_t K, int64_t N, int64_t E, int64_t group, int nproj, int nt);
moe_status launch_fwd_stream(ProjParams p, int nproj, bool bf16_mma, int nt, void *ws, size_t ws_bytes,
                             cudaStream_t st);
bool tc_available();
bool tc_fits(const ProjParams &p);
bool tc_bwd_fits(const BwdParams &p);
moe_status launch_fwd_tc(const ProjParams &p, int nproj, bool bf16_mma, cudaStream_t st);
moe_status launch_bwd_tc(const BwdParams &p, int nproj, bool bf16_mma, cudaStream_t st);
bool tc2_fits(const ProjParams &p);
bool tc2_bwd_fits(const BwdParams &p);
moe_status launch_bwd_tc2(const BwdParams &p, int nproj, bool bf16_mma, cudaStream_t st);
moe_status launch_fwd_tc2(const ProjParams &p, int nproj, bool bf16_mma, cudaStream_t st);
moe_status launch_act_to_f16(const void *src, void *dst, int64_t elems, int32_t *status, cudaStream_t st);

}  // namespace moe
