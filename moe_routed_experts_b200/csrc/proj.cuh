// Parameters of the grouped AWQ projection kernels (both tile paths).
#pragma once

#include "common.cuh"

namespace moe {

struct ProjParams {
  const uint16_t *x;  // [A, K] activations
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
};

// Final values of 8 consecutive output columns n0.. of row `row` of local
// expert e from FP32 sums (gate sums g, up sums u for the pair): bias, one
// rounding to the activation dtype, SwiGLU from the rounded G and U.
template <int NPROJ>
__device__ __forceinline__ void finish8(const ProjParams &p, int e, int64_t row, int64_t n0, const float *g,
                                        const float *u) {
  uint32_t o[4];
  if (NPROJ == 2) {
    uint32_t og[4], ou[4];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      float gv[2], uv[2];
#pragma unroll
      for (int d = 0; d < 2; ++d) {
        gv[d] = g[i + d];
        uv[d] = u[i + d];
        if (p.bias[0]) gv[d] += ld_as_float(p.bias[0], p.bias_dt, (int64_t)e * p.N + n0 + i + d);
        if (p.bias[1]) uv[d] += ld_as_float(p.bias[1], p.bias_dt, (int64_t)e * p.N + n0 + i + d);
      }
      const uint16_t gb0 = f32_to_bits(gv[0], p.act_dt), gb1 = f32_to_bits(gv[1], p.act_dt);
      const uint16_t ub0 = f32_to_bits(uv[0], p.act_dt), ub1 = f32_to_bits(uv[1], p.act_dt);
      const float g0 = bits_to_f32(gb0, p.act_dt), g1 = bits_to_f32(gb1, p.act_dt);
      const float x0 = bits_to_f32(ub0, p.act_dt), x1 = bits_to_f32(ub1, p.act_dt);
      const float h0 = g0 / (1.f + expf(-g0)) * x0, h1 = g1 / (1.f + expf(-g1)) * x1;
      og[i / 2] = uint32_t(gb0) | (uint32_t(gb1) << 16);
      ou[i / 2] = uint32_t(ub0) | (uint32_t(ub1) << 16);
      o[i / 2] = uint32_t(f32_to_bits(h0, p.act_dt)) | (uint32_t(f32_to_bits(h1, p.act_dt)) << 16);
    }
    if (p.gout) *reinterpret_cast<uint4 *>(p.gout + row * p.N + n0) = make_uint4(og[0], og[1], og[2], og[3]);
    if (p.uout) *reinterpret_cast<uint4 *>(p.uout + row * p.N + n0) = make_uint4(ou[0], ou[1], ou[2], ou[3]);
  } else {
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      float yv[2];
#pragma unroll
      for (int d = 0; d < 2; ++d) {
        yv[d] = g[i + d];
        if (p.bias[0]) yv[d] += ld_as_float(p.bias[0], p.bias_dt, (int64_t)e * p.N + n0 + i + d);
      }
      o[i / 2] = uint32_t(f32_to_bits(yv[0], p.act_dt)) | (uint32_t(f32_to_bits(yv[1], p.act_dt)) << 16);
    }
  }
  *reinterpret_cast<uint4 *>(p.out + row * p.N + n0) = make_uint4(o[0], o[1], o[2], o[3]);
}

void launch_fwd_mma(const ProjParams &p, int nproj, bool bf16_mma, int nt, cudaStream_t st);
void launch_bwd_mma(const BwdParams &p, int nproj, bool bf16_mma, int nt, cudaStream_t st);
void launch_dump(const int32_t *qw, const int32_t *qz, const uint16_t *sc, int64_t K, int64_t N, int group,
                 uint16_t *out, int mode, bool bf16_mma, cudaStream_t st);
struct StreamPlan {
  bool fits;      // the streaming tile can run this shape
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

}  // namespace moe
