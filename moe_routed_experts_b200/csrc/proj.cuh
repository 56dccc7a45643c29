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
moe_status launch_fwd_tc(const ProjParams &p, int nproj, bool bf16_mma, cudaStream_t st);
moe_status launch_bwd_tc(const BwdParams &p, int nproj, bool bf16_mma, cudaStream_t st);

}  // namespace moe
