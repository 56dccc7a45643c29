// Host entry points of the grouped AWQ projections, argument validation,
// error strings and the projection-path knob.
#include <stdarg.h>
#include <stdio.h>

#include <atomic>

#include "proj.cuh"

namespace moe {

static thread_local char g_err[1024] = "no error";

moe_status set_error(moe_status s, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

moe_status check_launch(const char *what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return MOE_OK;
}

int num_sms() {
  static std::atomic<int> cached{0};
  int v = cached.load();
  if (v > 0) return v;
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  cached.store(n);
  return n;
}

static std::atomic<int> g_path{0};

// All tile paths hold the same operation.  The warp-level one is chosen when
// the average batch per expert is too small to fill a 128-row tcgen05 tile,
// the CTA-pair one when experts average 384 rows or more (a 256-row tile is
// then at most a third empty on average), and a shape a tcgen05 tile does
// not take (tc_fits / tc2_fits) falls to the next path down.
static int choose_path(int64_t A, int64_t E) {
  int forced = g_path.load();
  if (forced >= 1 && forced <= 3) return forced;
  if (!tc_available()) return 1;
  if (A >= 384 * E) return 3;
  return (A >= 32 * E) ? 2 : 1;
}

// The tcgen05 forward tile the chosen path runs for this shape: 3 (CTA
// pair), 2 (single CTA), or 0 when neither takes it.
static int fwd_tc_kind(int path, const ProjParams &p) {
  if (path == 3 && tc2_fits(p)) return 3;
  if (path >= 2 && tc_fits(p)) return 2;
  return 0;
}

// Bytes of an F16 copy of `rows` x `cols` BF16 values (16-byte multiple).
static size_t conv_bytes(int64_t rows, int64_t cols) { return ((size_t)rows * cols * 2 + 255) & ~size_t(255); }

// A tcgen05 tile with F16 coefficients and BF16 inputs: when the workspace
// holds it, make the F16 copy of the inputs once (src -> ws) and return it,
// else return NULL (the tile converts in place).
static const uint16_t *maybe_convert(const void *src, moe_dtype in_dt, moe_dtype scale_dt, int64_t rows, int64_t cols,
                                     void *ws, size_t ws_bytes, int32_t *status, cudaStream_t st, moe_status *err) {
  *err = MOE_OK;
  if (in_dt != MOE_BF16 || scale_dt != MOE_F16 || !ws || ws_bytes < conv_bytes(rows, cols) || !aligned16(ws))
    return nullptr;
  *err = launch_act_to_f16(src, ws, rows * cols, status, st);
  return *err == MOE_OK ? static_cast<const uint16_t *>(ws) : nullptr;
}

static moe_status run_fwd_tc(int kind, ProjParams p, int nproj, bool bf, moe_dtype scale_dt, void *ws,
                             size_t ws_bytes, cudaStream_t st) {
  moe_status err;
  const uint16_t *conv = maybe_convert(p.x, (moe_dtype)p.act_dt, scale_dt, p.gather ? p.T : p.A, p.K, ws, ws_bytes,
                                       p.status, st, &err);
  if (err != MOE_OK) return err;
  if (conv) {
    p.x = conv;
    p.preconv = 1;
  }
  return kind == 3 ? launch_fwd_tc2(p, nproj, bf, st) : launch_fwd_tc(p, nproj, bf, st);
}

// Token columns per warp-level tile: 16 when experts average >= 12 rows.
static int small_tile_tokens(int64_t A, int64_t E) { return A >= 12 * E ? 2 : 1; }

static moe_status check_payload_geom(const char *fn, int64_t A, int64_t K, int64_t N, int64_t E, int64_t group,
                                     moe_dtype act_dt, moe_dtype scale_dt) {
  if (act_dt != MOE_F16 && act_dt != MOE_BF16)
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "%s: activations must be F16 or BF16", fn);
  if (scale_dt == MOE_F32)
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "%s: FP32 scales are not run by this library", fn);
  if (scale_dt != MOE_F16 && scale_dt != MOE_BF16)
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "%s: bad scale dtype %d", fn, (int)scale_dt);
  if (A < 0 || E < 1 || E > MOE_MAX_EXPERTS || K < 16 || N < 8)
    return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: bad sizes A=%lld K=%lld N=%lld E=%lld", fn, (long long)A,
                     (long long)K, (long long)N, (long long)E);
  if (N % 8 != 0) return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: N=%lld not divisible by 8", fn, (long long)N);
  if (group < 16 || group % 16 != 0 || K % group != 0)
    return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: group=%lld must be a multiple of 16 dividing K=%lld", fn,
                     (long long)group, (long long)K);
  if (A > INT32_MAX) return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: A exceeds int32 row offsets", fn);
  return MOE_OK;
}

static moe_status check_ptrs(const char *fn, std::initializer_list<const void *> must, std::initializer_list<const void *> al16) {
  for (const void *q : must)
    if (!q) return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: NULL tensor pointer", fn);
  for (const void *q : al16)
    if (q && !aligned16(q)) return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: tensor not 16-byte aligned", fn);
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" const char *moe_last_error_string(void) { return g_err; }

extern "C" const char *moe_version(void) { return "moe_awq 0.1.0 sm_100a"; }

extern "C" int32_t moe_set_projection_path(int32_t path) {
  if (path < 0 || path > 3) return -1;
  if (path >= 2 && !tc_available()) return -1;
  return g_path.exchange(path);
}

extern "C" size_t awq_projection_workspace_size_dt(int64_t A, int64_t K, int64_t N, int64_t E, int64_t group_size,
                                                   int32_t nproj, moe_dtype act_dtype, moe_dtype scale_dtype) {
  if (A <= 0 || E < 1 || K < 16 || N < 8 || group_size < 16 || (nproj != 1 && nproj != 2)) return 0;
  ProjParams probe{};
  probe.A = A;
  probe.K = K;
  probe.N = N;
  probe.E = (int)E;
  probe.group = (int)group_size;
  if (fwd_tc_kind(choose_path(A, E), probe))
    return (act_dtype == MOE_BF16 && scale_dtype == MOE_F16) ? conv_bytes(A, K) : 0;
  const StreamPlan pl = stream_plan(A, K, N, E, group_size, nproj, small_tile_tokens(A, E));
  return pl.fits ? pl.bytes : 0;
}

extern "C" size_t awq_projection_workspace_size(int64_t A, int64_t K, int64_t N, int64_t E, int64_t group_size,
                                                int32_t nproj) {
  return awq_projection_workspace_size_dt(A, K, N, E, group_size, nproj, MOE_BF16, MOE_F16);
}

extern "C" size_t awq_input_backward_workspace_size(int64_t A, int64_t N, int64_t K, int64_t E, int64_t group_size,
                                                    int32_t nproj, moe_dtype grad_dtype, moe_dtype scale_dtype) {
  if (A <= 0 || E < 1 || K < 16 || N < 8 || group_size < 16 || (nproj != 1 && nproj != 2)) return 0;
  if (grad_dtype != MOE_BF16 || scale_dtype != MOE_F16 || choose_path(A, E) < 2) return 0;
  return (size_t)nproj * conv_bytes(A, N);
}

// Gate/up projections of expert-sorted rows that are read from `values`
// (gather == NULL) or as x[gather[r]] (x has T rows).
static moe_status gate_up_impl(const char *fn, const void *x, const int32_t *gather, int64_t T, moe_dtype act_dtype,
                               int64_t A, int64_t H, int64_t I, const int32_t *offsets, int64_t E,
                               const int32_t *qweight_gate, const int32_t *qzeros_gate, const void *scales_gate,
                               const void *bias_gate, const int32_t *qweight_up, const int32_t *qzeros_up,
                               const void *scales_up, const void *bias_up, moe_dtype scale_dtype,
                               moe_dtype bias_dtype, int64_t group_size, void *h, moe_dtype h_dtype, void *gate_out,
                               void *up_out, moe_dtype out_dtype, void *workspace, size_t workspace_bytes,
                               int32_t *device_status, void *stream) {
  moe_status s = check_payload_geom(fn, A, H, I, E, group_size, act_dtype, scale_dtype);
  if (s != MOE_OK) return s;
  if ((out_dtype != MOE_F16 && out_dtype != MOE_BF16) || (h_dtype != MOE_F16 && h_dtype != MOE_BF16))
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "%s: output dtypes must be F16 or BF16", fn);
  if ((bias_gate || bias_up) && !valid_dtype(bias_dtype))
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "%s: bad bias dtype", fn);
  if (gather && T < 1) return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: T=%lld rows of x", fn, (long long)T);
  if (A == 0) return MOE_OK;
  s = check_ptrs(fn, {x, offsets, qweight_gate, qzeros_gate, scales_gate, qweight_up, qzeros_up, scales_up, h},
                 {x, scales_gate, scales_up, h, gate_out, up_out, qweight_gate, qweight_up, bias_gate, bias_up});
  if (s != MOE_OK) return s;
  ProjParams p{};
  p.x = static_cast<const uint16_t *>(x);
  p.gather = gather;
  p.T = gather ? T : A;
  p.act_dt = act_dtype;
  p.odt = out_dtype;
  p.hdt = h_dtype;
  p.A = A;
  p.K = H;
  p.N = I;
  p.offsets = offsets;
  p.E = (int)E;
  p.qw[0] = qweight_gate;
  p.qw[1] = qweight_up;
  p.qz[0] = qzeros_gate;
  p.qz[1] = qzeros_up;
  p.sc[0] = static_cast<const uint16_t *>(scales_gate);
  p.sc[1] = static_cast<const uint16_t *>(scales_up);
  p.bias[0] = bias_gate;
  p.bias[1] = bias_up;
  p.bias_dt = bias_dtype;
  p.group = (int)group_size;
  p.out = static_cast<uint16_t *>(h);
  p.gout = static_cast<uint16_t *>(gate_out);
  p.uout = static_cast<uint16_t *>(up_out);
  p.status = device_status;
  cudaStream_t st = as_stream(stream);
  const bool bf = scale_dtype == MOE_BF16;
  const int kind = fwd_tc_kind(choose_path(A, E), p);
  if (kind) return run_fwd_tc(kind, p, 2, bf, scale_dtype, workspace, workspace_bytes, st);
  const int nt = small_tile_tokens(A, E);
  if (stream_plan(A, H, I, E, group_size, 2, nt).fits) return launch_fwd_stream(p, 2, bf, nt, workspace, workspace_bytes, st);
  launch_fwd_mma(p, 2, bf, nt, st);
  return check_launch(fn);
}

extern "C" moe_status awq_grouped_gate_up_swiglu(
    const void *values, moe_dtype act_dtype, int64_t A, int64_t H, int64_t I, const int32_t *offsets, int64_t E,
    const int32_t *qweight_gate, const int32_t *qzeros_gate, const void *scales_gate, const void *bias_gate,
    const int32_t *qweight_up, const int32_t *qzeros_up, const void *scales_up, const void *bias_up,
    moe_dtype scale_dtype, moe_dtype bias_dtype, int64_t group_size, void *h, void *gate_out, void *up_out,
    void *workspace, size_t workspace_bytes, int32_t *device_status, void *stream) {
  return gate_up_impl("awq_grouped_gate_up_swiglu", values, nullptr, A, act_dtype, A, H, I, offsets, E, qweight_gate,
                      qzeros_gate, scales_gate, bias_gate, qweight_up, qzeros_up, scales_up, bias_up, scale_dtype,
                      bias_dtype, group_size, h, act_dtype, gate_out, up_out, act_dtype, workspace, workspace_bytes,
                      device_status, stream);
}

extern "C" moe_status awq_grouped_gate_up_swiglu_dt(
    const void *values, moe_dtype act_dtype, int64_t A, int64_t H, int64_t I, const int32_t *offsets, int64_t E,
    const int32_t *qweight_gate, const int32_t *qzeros_gate, const void *scales_gate, const void *bias_gate,
    const int32_t *qweight_up, const int32_t *qzeros_up, const void *scales_up, const void *bias_up,
    moe_dtype scale_dtype, moe_dtype bias_dtype, int64_t group_size, void *h, moe_dtype h_dtype, void *gate_out,
    void *up_out, moe_dtype out_dtype, void *workspace, size_t workspace_bytes, int32_t *device_status,
    void *stream) {
  return gate_up_impl("awq_grouped_gate_up_swiglu", values, nullptr, A, act_dtype, A, H, I, offsets, E, qweight_gate,
                      qzeros_gate, scales_gate, bias_gate, qweight_up, qzeros_up, scales_up, bias_up, scale_dtype,
                      bias_dtype, group_size, h, h_dtype, gate_out, up_out, out_dtype, workspace, workspace_bytes,
                      device_status, stream);
}

extern "C" moe_status awq_grouped_gate_up_swiglu_gather(
    const void *x, moe_dtype act_dtype, int64_t T, const int32_t *src_token, int64_t A, int64_t H, int64_t I,
    const int32_t *offsets, int64_t E, const int32_t *qweight_gate, const int32_t *qzeros_gate,
    const void *scales_gate, const void *bias_gate, const int32_t *qweight_up, const int32_t *qzeros_up,
    const void *scales_up, const void *bias_up, moe_dtype scale_dtype, moe_dtype bias_dtype, int64_t group_size,
    void *h, void *gate_out, void *up_out, void *workspace, size_t workspace_bytes, int32_t *device_status,
    void *stream) {
  const char *fn = "awq_grouped_gate_up_swiglu_gather";
  if (A > 0 && !src_token) return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: src_token is NULL", fn);
  return gate_up_impl(fn, x, src_token, T, act_dtype, A, H, I, offsets, E, qweight_gate, qzeros_gate, scales_gate,
                      bias_gate, qweight_up, qzeros_up, scales_up, bias_up, scale_dtype, bias_dtype, group_size, h,
                      act_dtype, gate_out, up_out, act_dtype, workspace, workspace_bytes, device_status, stream);
}

extern "C" moe_status awq_grouped_gate_up_swiglu_gather_dt(
    const void *x, moe_dtype act_dtype, int64_t T, const int32_t *src_token, int64_t A, int64_t H, int64_t I,
    const int32_t *offsets, int64_t E, const int32_t *qweight_gate, const int32_t *qzeros_gate,
    const void *scales_gate, const void *bias_gate, const int32_t *qweight_up, const int32_t *qzeros_up,
    const void *scales_up, const void *bias_up, moe_dtype scale_dtype, moe_dtype bias_dtype, int64_t group_size,
    void *h, moe_dtype h_dtype, void *gate_out, void *up_out, moe_dtype out_dtype, void *workspace,
    size_t workspace_bytes, int32_t *device_status, void *stream) {
  const char *fn = "awq_grouped_gate_up_swiglu_gather";
  if (A > 0 && !src_token) return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: src_token is NULL", fn);
  return gate_up_impl(fn, x, src_token, T, act_dtype, A, H, I, offsets, E, qweight_gate, qzeros_gate, scales_gate,
                      bias_gate, qweight_up, qzeros_up, scales_up, bias_up, scale_dtype, bias_dtype, group_size, h,
                      h_dtype, gate_out, up_out, out_dtype, workspace, workspace_bytes, device_status, stream);
}

extern "C" moe_status awq_grouped_down_dt(const void *input, moe_dtype act_dtype, int64_t A, int64_t K, int64_t N,
                                          const int32_t *offsets, int64_t E, const int32_t *qweight,
                                          const int32_t *qzeros, const void *scales, const void *bias,
                                          moe_dtype scale_dtype, moe_dtype bias_dtype, int64_t group_size,
                                          void *output, moe_dtype out_dtype, void *workspace,
                                          size_t workspace_bytes, int32_t *device_status, void *stream) {
  const char *fn = "awq_grouped_down";
  moe_status s = check_payload_geom(fn, A, K, N, E, group_size, act_dtype, scale_dtype);
  if (s != MOE_OK) return s;
  if (out_dtype != MOE_F16 && out_dtype != MOE_BF16)
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "%s: out_dtype must be F16 or BF16", fn);
  if (bias && !valid_dtype(bias_dtype)) return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "%s: bad bias dtype", fn);
  if (A == 0) return MOE_OK;
  s = check_ptrs(fn, {input, offsets, qweight, qzeros, scales, output}, {input, scales, output, qweight, bias});
  if (s != MOE_OK) return s;
  ProjParams p{};
  p.x = static_cast<const uint16_t *>(input);
  p.act_dt = act_dtype;
  p.odt = out_dtype;
  p.hdt = out_dtype;
  p.A = A;
  p.K = K;
  p.N = N;
  p.offsets = offsets;
  p.E = (int)E;
  p.qw[0] = p.qw[1] = qweight;
  p.qz[0] = p.qz[1] = qzeros;
  p.sc[0] = p.sc[1] = static_cast<const uint16_t *>(scales);
  p.bias[0] = p.bias[1] = bias;
  p.bias_dt = bias_dtype;
  p.group = (int)group_size;
  p.out = static_cast<uint16_t *>(output);
  p.status = device_status;
  cudaStream_t st = as_stream(stream);
  const bool bf = scale_dtype == MOE_BF16;
  const int kind = fwd_tc_kind(choose_path(A, E), p);
  if (kind) return run_fwd_tc(kind, p, 1, bf, scale_dtype, workspace, workspace_bytes, st);
  const int nt = small_tile_tokens(A, E);
  if (stream_plan(A, K, N, E, group_size, 1, nt).fits) return launch_fwd_stream(p, 1, bf, nt, workspace, workspace_bytes, st);
  launch_fwd_mma(p, 1, bf, nt, st);
  return check_launch(fn);
}

extern "C" moe_status awq_grouped_down(const void *input, moe_dtype act_dtype, int64_t A, int64_t K, int64_t N,
                                       const int32_t *offsets, int64_t E, const int32_t *qweight,
                                       const int32_t *qzeros, const void *scales, const void *bias,
                                       moe_dtype scale_dtype, moe_dtype bias_dtype, int64_t group_size,
                                       void *output, void *workspace, size_t workspace_bytes,
                                       int32_t *device_status, void *stream) {
  return awq_grouped_down_dt(input, act_dtype, A, K, N, offsets, E, qweight, qzeros, scales, bias, scale_dtype,
                             bias_dtype, group_size, output, act_dtype, workspace, workspace_bytes, device_status,
                             stream);
}

extern "C" moe_status awq_input_backward_dt(const void *grad, moe_dtype grad_dtype, int64_t A, int64_t N, int64_t K,
                                            const int32_t *offsets, int64_t E, const int32_t *qweight,
                                            const int32_t *qzeros, const void *scales, moe_dtype scale_dtype,
                                            int64_t group_size, const void *grad2, const int32_t *qweight2,
                                            const int32_t *qzeros2, const void *scales2, void *dinput,
                                            moe_dtype dinput_dtype, void *workspace, size_t workspace_bytes,
                                            int32_t *device_status, void *stream) {
  const char *fn = "awq_input_backward";
  moe_status s = check_payload_geom(fn, A, K, N, E, group_size, grad_dtype, scale_dtype);
  if (s != MOE_OK) return s;
  if (dinput_dtype != MOE_F16 && dinput_dtype != MOE_BF16)
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "%s: dinput_dtype must be F16 or BF16", fn);
  if (A == 0) return MOE_OK;
  s = check_ptrs(fn, {grad, offsets, qweight, qzeros, scales, dinput}, {grad, scales, dinput, grad2, scales2});
  if (s != MOE_OK) return s;
  if (grad2) {
    s = check_ptrs(fn, {qweight2, qzeros2, scales2}, {});
    if (s != MOE_OK) return s;
  }
  BwdParams p{};
  p.grad[0] = static_cast<const uint16_t *>(grad);
  p.grad[1] = static_cast<const uint16_t *>(grad2 ? grad2 : grad);
  p.gdt = grad_dtype;
  p.odt = dinput_dtype;
  p.A = A;
  p.N = N;
  p.K = K;
  p.offsets = offsets;
  p.E = (int)E;
  p.qw[0] = qweight;
  p.qz[0] = qzeros;
  p.sc[0] = static_cast<const uint16_t *>(scales);
  p.qw[1] = grad2 ? qweight2 : qweight;
  p.qz[1] = grad2 ? qzeros2 : qzeros;
  p.sc[1] = static_cast<const uint16_t *>(grad2 ? scales2 : scales);
  p.group = (int)group_size;
  p.out = static_cast<uint16_t *>(dinput);
  p.status = device_status;
  cudaStream_t st = as_stream(stream);
  const bool bf = scale_dtype == MOE_BF16;
  const int nproj = grad2 ? 2 : 1;
  const int path = choose_path(A, E);
  const int kind = (path == 3 && tc2_bwd_fits(p)) ? 3 : (path >= 2 && tc_bwd_fits(p)) ? 2 : 0;
  if (kind) {
    // F16 copies of the gradients, once, when the workspace holds both
    const size_t one = conv_bytes(A, N);
    if (grad_dtype == MOE_BF16 && scale_dtype == MOE_F16 && workspace && aligned16(workspace) &&
        workspace_bytes >= (size_t)nproj * one) {
      char *w = static_cast<char *>(workspace);
      s = launch_act_to_f16(grad, w, A * N, device_status, st);
      if (s == MOE_OK && grad2) s = launch_act_to_f16(grad2, w + one, A * N, device_status, st);
      if (s != MOE_OK) return s;
      p.grad[0] = reinterpret_cast<const uint16_t *>(w);
      p.grad[1] = reinterpret_cast<const uint16_t *>(grad2 ? w + one : w);
      p.preconv = 1;
    }
    return kind == 3 ? launch_bwd_tc2(p, nproj, bf, st) : launch_bwd_tc(p, nproj, bf, st);
  }
  launch_bwd_mma(p, nproj, bf, A >= 12 * E ? 2 : 1, st);
  return check_launch(fn);
}

extern "C" moe_status awq_input_backward(const void *grad, moe_dtype grad_dtype, int64_t A, int64_t N, int64_t K,
                                         const int32_t *offsets, int64_t E, const int32_t *qweight,
                                         const int32_t *qzeros, const void *scales, moe_dtype scale_dtype,
                                         int64_t group_size, const void *grad2, const int32_t *qweight2,
                                         const int32_t *qzeros2, const void *scales2, void *dinput,
                                         void *workspace, size_t workspace_bytes, int32_t *device_status,
                                         void *stream) {
  return awq_input_backward_dt(grad, grad_dtype, A, N, K, offsets, E, qweight, qzeros, scales, scale_dtype,
                               group_size, grad2, qweight2, qzeros2, scales2, dinput, grad_dtype, workspace,
                               workspace_bytes, device_status, stream);
}

extern "C" moe_status awq_dequant_coefficients(const int32_t *qweight, const int32_t *qzeros, const void *scales,
                                               moe_dtype scale_dtype, int64_t K, int64_t N, int64_t group_size,
                                               int32_t pairing, uint16_t *coefficients, void *stream) {
  const char *fn = "awq_dequant_coefficients";
  moe_status s = check_payload_geom(fn, 0, K, N, 1, group_size, MOE_BF16, scale_dtype);
  if (s != MOE_OK) return s;
  s = check_ptrs(fn, {qweight, qzeros, scales, coefficients}, {scales});
  if (s != MOE_OK) return s;
  if (pairing != 0 && pairing != 1) return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: pairing must be 0 or 1", fn);
  launch_dump(qweight, qzeros, static_cast<const uint16_t *>(scales), K, N, (int)group_size, coefficients, pairing,
              scale_dtype == MOE_BF16, as_stream(stream));
  return check_launch(fn);
}
