// Combine, its VJP, the COPY-dispatch VJP and the SwiGLU VJP.
//
// ruda-tensor 0.21.38, src/moe_exchange.rs:
//   moe_combine           -- per token, ascending expert-ID combine of the
//                            expert rows with the FP32 weights;
//   moe_combine_backward  -- requested expert-row and FP32 weight VJPs
//                            (MoeCombineSelection / MoeCombineBackward);
//   moe_dispatch_backward -- the COPY VJP sums the selected row seeds without
//                            applying the routing weights again.
// ruda-tensor 0.21.34, src/packed_experts.rs, packed_swiglu_input_backward --
//   the SwiGLU step of the input VJP.
//
// One CTA per token: warp 0 orders the token's k selections by expert ID
// (k <= 32, one lane each), then every thread accumulates 8 columns in FP32
// from +0 in that order and rounds once.  Memory-bound: each kernel reads
// and writes each row once with 16-byte accesses.
#include "common.cuh"

namespace moe {

constexpr int kCombThreads = 256;

struct CombineParams {
  const void *y;  // [A, H] rows (or dvalues)
  int dt;
  int64_t A;
  const float *weights;  // NULL: plain sum (COPY VJP)
  const uint32_t *selected;
  const int32_t *row_of;
  int64_t T, H;
  int k;
  void *out;
  int32_t *status;
};

// Fills ord_row/ord_w (shared) with the token's rows in ascending expert ID;
// invalid rows get -1.
__device__ __forceinline__ void order_token(const uint32_t *sel, const int32_t *row_of, const float *w,
                                            int k, int64_t A, int64_t t, int32_t *ord_row, float *ord_w,
                                            int32_t *status) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    uint32_t id = lane < k ? sel[t * k + lane] : 0xFFFFFFFFu;
    int32_t r = lane < k ? row_of[t * k + lane] : -1;
    float wv = (lane < k && w) ? w[t * k + lane] : 1.f;
    int pos = 0;
    for (int j = 0; j < k; ++j) {
      uint32_t oj = __shfl_sync(0xffffffffu, id, j);
      pos += (oj < id || (oj == id && j < lane)) ? 1 : 0;
    }
    if (lane < k) {
      if (r < 0 || (int64_t)r >= A) {
        report(status, MOE_DEVICE_ERR_ROW_RANGE);
        r = -1;
      }
      ord_row[pos] = r;
      ord_w[pos] = wv;
    }
  }
  __syncthreads();
}

template <bool VEC>
__global__ void __launch_bounds__(kCombThreads) combine_kernel(CombineParams p) {
  pdl_enter();  // programmatic dependent launch: the previous kernel is done
  __shared__ int32_t ord_row[MOE_MAX_TOP_K];
  __shared__ float ord_w[MOE_MAX_TOP_K];
  const int64_t t = blockIdx.x;
  order_token(p.selected, p.row_of, p.weights, p.k, p.A, t, ord_row, ord_w, p.status);
  const uint16_t *y = static_cast<const uint16_t *>(p.y);
  uint16_t *out = static_cast<uint16_t *>(p.out);
  if (VEC) {
    for (int64_t c0 = (int64_t)threadIdx.x * 8; c0 < p.H; c0 += (int64_t)blockDim.x * 8) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      for (int j0 = 0; j0 < p.k; j0 += 8) {
        // issue up to 8 row loads before summing them in ascending-ID order
        uint4 v[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int32_t r = j0 + jj < p.k ? ord_row[j0 + jj] : -1;
          v[jj] = r >= 0 ? *reinterpret_cast<const uint4 *>(y + (int64_t)r * p.H + c0) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          if (j0 + jj >= p.k || ord_row[j0 + jj] < 0) continue;
          const float wv = ord_w[j0 + jj];
          const uint32_t u[4] = {v[jj].x, v[jj].y, v[jj].z, v[jj].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float lo = bits_to_f32(uint16_t(u[i] & 0xFFFF), p.dt), hi = bits_to_f32(uint16_t(u[i] >> 16), p.dt);
            if (p.weights) {
              acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(wv, lo));
              acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(wv, hi));
            } else {
              acc[2 * i] = __fadd_rn(acc[2 * i], lo);
              acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], hi);
            }
          }
        }
      }
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o[i] = uint32_t(f32_to_bits(acc[2 * i], p.dt)) | (uint32_t(f32_to_bits(acc[2 * i + 1], p.dt)) << 16);
      *reinterpret_cast<uint4 *>(out + t * p.H + c0) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  } else {
    for (int64_t c = threadIdx.x; c < p.H; c += blockDim.x) {
      float acc = 0.f;
      for (int j = 0; j < p.k; ++j) {
        const int32_t r = ord_row[j];
        if (r < 0) continue;
        float v = bits_to_f32(y[(int64_t)r * p.H + c], p.dt);
        acc = p.weights ? __fadd_rn(acc, __fmul_rn(ord_w[j], v)) : __fadd_rn(acc, v);
      }
      out[t * p.H + c] = f32_to_bits(acc, p.dt);
    }
  }
}

struct CombineBwdParams {
  const void *d_out;
  const void *y;
  int dt;
  int64_t A;
  const float *weights;
  const int32_t *row_of;
  int64_t T, H;
  int k;
  void *dy;
  float *dweights;
  int32_t *status;
  int odt;  // dtype of dy
};

// v rounded to dtype dt.  With chk (BF16-range values written as F16), a
// value that is not +-inf but becomes inf or NaN in F16 sets bad, the rule
// of the BF16 -> F16 input conversion.
__device__ __forceinline__ uint16_t f32_to_bits_chk(float v, int dt, bool chk, uint32_t &bad) {
  const uint16_t r = f32_to_bits(v, dt);
  if (chk && (r & 0x7C00u) == 0x7C00u && !isinf(v)) bad = 1;
  return r;
}

// One CTA per token.  dy rows are written with one rounding of the exact
// FP32 product; the dots are reduced in a fixed tree (per thread, warp, CTA).
// VEC: 8 columns per thread and access (16-byte loads and stores).
template <bool VEC>
__global__ void __launch_bounds__(kCombThreads) combine_bwd_kernel(CombineBwdParams p) {
  __shared__ float red[kCombThreads / 32][MOE_MAX_TOP_K];
  const int64_t t = blockIdx.x;
  const uint16_t *g = static_cast<const uint16_t *>(p.d_out);
  const uint16_t *y = static_cast<const uint16_t *>(p.y);
  uint16_t *dy = static_cast<uint16_t *>(p.dy);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool chk = p.odt == MOE_F16 && p.dt == MOE_BF16;
  uint32_t bad = 0;
  for (int j = 0; j < p.k; ++j) {
    int32_t r = p.row_of[t * p.k + j];
    const bool ok = r >= 0 && (int64_t)r < p.A;
    if (!ok && threadIdx.x == 0) report(p.status, MOE_DEVICE_ERR_ROW_RANGE);
    const float w = p.weights[t * p.k + j];
    float dot = 0.f;
    if (ok && VEC) {
      for (int64_t c0 = (int64_t)threadIdx.x * 8; c0 < p.H; c0 += (int64_t)blockDim.x * 8) {
        const uint4 gv = *reinterpret_cast<const uint4 *>(g + t * p.H + c0);
        const uint32_t gu[4] = {gv.x, gv.y, gv.z, gv.w};
        float gf[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          gf[2 * i] = bits_to_f32(uint16_t(gu[i] & 0xFFFF), p.dt);
          gf[2 * i + 1] = bits_to_f32(uint16_t(gu[i] >> 16), p.dt);
        }
        if (dy) {
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            o[i] = uint32_t(f32_to_bits_chk(__fmul_rn(w, gf[2 * i]), p.odt, chk, bad)) |
                   (uint32_t(f32_to_bits_chk(__fmul_rn(w, gf[2 * i + 1]), p.odt, chk, bad)) << 16);
          *reinterpret_cast<uint4 *>(dy + (int64_t)r * p.H + c0) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        if (p.dweights) {
          const uint4 yv = *reinterpret_cast<const uint4 *>(y + (int64_t)r * p.H + c0);
          const uint32_t yu[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            dot = fmaf(gf[2 * i], bits_to_f32(uint16_t(yu[i] & 0xFFFF), p.dt), dot);
            dot = fmaf(gf[2 * i + 1], bits_to_f32(uint16_t(yu[i] >> 16), p.dt), dot);
          }
        }
      }
    } else if (ok) {
      for (int64_t c = threadIdx.x; c < p.H; c += blockDim.x) {
        float gv = bits_to_f32(g[t * p.H + c], p.dt);
        if (dy) dy[(int64_t)r * p.H + c] = f32_to_bits_chk(__fmul_rn(w, gv), p.odt, chk, bad);
        if (p.dweights) dot = fmaf(gv, bits_to_f32(y[(int64_t)r * p.H + c], p.dt), dot);
      }
    }
    if (p.dweights) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if (lane == 0) red[warp][j] = dot;
    }
  }
  if (bad) report(p.status, MOE_DEVICE_ERR_ACT_RANGE);
  if (!p.dweights) return;
  __syncthreads();
  if (threadIdx.x < p.k) {
    float s = 0.f;
    for (int w = 0; w < kCombThreads / 32; ++w) s += red[w][threadIdx.x];
    p.dweights[t * p.k + threadIdx.x] = s;
  }
}

struct SwigluBwdParams {
  const uint16_t *dh, *G, *U;
  uint16_t *dG, *dU;
  int dt;
  int64_t n;
  int vec;  // all five tensors 16-byte aligned: 8 elements per access
  int odt;  // dtype of dG and dU
  int32_t *status;
};

// sigma = 1/(1+e^-G); dG = dh U sigma (1 + G (1 - sigma)), dU = dh G sigma, each
// rounded once.  Fast exponential and division: few-ulp FP32 error, far below
// one rounding of the 16-bit result.  8 elements per thread and access.
__device__ __forceinline__ void swiglu_bwd1(float d, float g, float u, float &dg, float &du) {
  const float s = __fdividef(1.f, 1.f + __expf(-g));
  dg = d * u * s * (1.f + g * (1.f - s));
  du = d * g * s;
}

__global__ void __launch_bounds__(256) swiglu_bwd_kernel(SwigluBwdParams p) {
  const int64_t n8 = p.vec ? p.n / 8 : 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const bool chk = p.odt == MOE_F16 && p.dt == MOE_BF16;
  uint32_t bad = 0;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < n8; v += stride) {
    const uint4 dv = reinterpret_cast<const uint4 *>(p.dh)[v];
    const uint4 gv = reinterpret_cast<const uint4 *>(p.G)[v];
    const uint4 uv = reinterpret_cast<const uint4 *>(p.U)[v];
    const uint32_t da[4] = {dv.x, dv.y, dv.z, dv.w}, ga[4] = {gv.x, gv.y, gv.z, gv.w}, ua[4] = {uv.x, uv.y, uv.z, uv.w};
    uint32_t og[4], ou[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float dg0, du0, dg1, du1;
      swiglu_bwd1(bits_to_f32(uint16_t(da[i] & 0xFFFF), p.dt), bits_to_f32(uint16_t(ga[i] & 0xFFFF), p.dt),
                  bits_to_f32(uint16_t(ua[i] & 0xFFFF), p.dt), dg0, du0);
      swiglu_bwd1(bits_to_f32(uint16_t(da[i] >> 16), p.dt), bits_to_f32(uint16_t(ga[i] >> 16), p.dt),
                  bits_to_f32(uint16_t(ua[i] >> 16), p.dt), dg1, du1);
      og[i] = uint32_t(f32_to_bits_chk(dg0, p.odt, chk, bad)) | (uint32_t(f32_to_bits_chk(dg1, p.odt, chk, bad)) << 16);
      ou[i] = uint32_t(f32_to_bits_chk(du0, p.odt, chk, bad)) | (uint32_t(f32_to_bits_chk(du1, p.odt, chk, bad)) << 16);
    }
    reinterpret_cast<uint4 *>(p.dG)[v] = make_uint4(og[0], og[1], og[2], og[3]);
    reinterpret_cast<uint4 *>(p.dU)[v] = make_uint4(ou[0], ou[1], ou[2], ou[3]);
  }
  // tail (n not a multiple of 8, or unaligned tensors)
  for (int64_t i = n8 * 8 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.n; i += stride) {
    float dg, du;
    swiglu_bwd1(bits_to_f32(p.dh[i], p.dt), bits_to_f32(p.G[i], p.dt), bits_to_f32(p.U[i], p.dt), dg, du);
    p.dG[i] = f32_to_bits_chk(dg, p.odt, chk, bad);
    p.dU[i] = f32_to_bits_chk(du, p.odt, chk, bad);
  }
  if (bad) report(p.status, MOE_DEVICE_ERR_ACT_RANGE);
}

static moe_status launch_combine(const CombineParams &p, cudaStream_t st, const char *what) {
  if (p.T == 0) return MOE_OK;
  const bool vec = aligned16(p.y) && aligned16(p.out) && p.H % 8 == 0;
  if (vec)
    launch_pdl(combine_kernel<true>, dim3((unsigned)p.T), dim3(kCombThreads), 0, st, p);
  else
    launch_pdl(combine_kernel<false>, dim3((unsigned)p.T), dim3(kCombThreads), 0, st, p);
  return check_launch(what);
}

static moe_status check_tk(const char *fn, int64_t T, int64_t H, int32_t k, int64_t A) {
  if (T < 0 || H < 1 || k < 1 || k > MOE_MAX_TOP_K || A < 0)
    return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: bad sizes T=%lld H=%lld top_k=%d A=%lld", fn, (long long)T,
                     (long long)H, k, (long long)A);
  if (T > INT32_MAX) return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: T too large", fn);
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_combine(const void *y, moe_dtype act_dtype, int64_t A, const float *weights,
                                  const uint32_t *selected_experts, const int32_t *row_of, int64_t T, int64_t H,
                                  int32_t top_k, void *out, int32_t *device_status, void *stream) {
  moe_status s = check_tk("moe_combine", T, H, top_k, A);
  if (s != MOE_OK) return s;
  if (act_dtype != MOE_F16 && act_dtype != MOE_BF16)
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "moe_combine: act_dtype must be F16 or BF16");
  if (T > 0 && (!y || !weights || !selected_experts || !row_of || !out))
    return set_error(MOE_ERR_INVALID_ARGUMENT, "moe_combine: NULL tensor pointer");
  CombineParams p{y, (int)act_dtype, A, weights, selected_experts, row_of, T, H, top_k, out, device_status};
  return launch_combine(p, as_stream(stream), "moe_combine");
}

extern "C" moe_status moe_dispatch_backward(const void *dvalues, moe_dtype act_dtype, int64_t A,
                                            const int32_t *row_of, const uint32_t *selected_experts, int64_t T,
                                            int64_t H, int32_t top_k, void *dx, int32_t *device_status,
                                            void *stream) {
  moe_status s = check_tk("moe_dispatch_backward", T, H, top_k, A);
  if (s != MOE_OK) return s;
  if (act_dtype != MOE_F16 && act_dtype != MOE_BF16)
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "moe_dispatch_backward: act_dtype must be F16 or BF16");
  if (T > 0 && (!dvalues || !selected_experts || !row_of || !dx))
    return set_error(MOE_ERR_INVALID_ARGUMENT, "moe_dispatch_backward: NULL tensor pointer");
  CombineParams p{dvalues, (int)act_dtype, A, nullptr, selected_experts, row_of, T, H, top_k, dx, device_status};
  return launch_combine(p, as_stream(stream), "moe_dispatch_backward");
}

extern "C" moe_status moe_combine_backward_dt(const void *d_out, const void *y, moe_dtype act_dtype, int64_t A,
                                              const float *weights, const int32_t *row_of, int64_t T, int64_t H,
                                              int32_t top_k, void *dy, moe_dtype dy_dtype, float *dweights,
                                              int32_t *device_status, void *stream) {
  moe_status s = check_tk("moe_combine_backward", T, H, top_k, A);
  if (s != MOE_OK) return s;
  if (act_dtype != MOE_F16 && act_dtype != MOE_BF16)
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "moe_combine_backward: act_dtype must be F16 or BF16");
  if (dy_dtype != MOE_F16 && dy_dtype != MOE_BF16)
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "moe_combine_backward: dy_dtype must be F16 or BF16");
  if (T == 0 || (!dy && !dweights)) return MOE_OK;
  if (!d_out || !weights || !row_of || (dweights && !y))
    return set_error(MOE_ERR_INVALID_ARGUMENT, "moe_combine_backward: NULL tensor pointer");
  CombineBwdParams p{d_out, y, (int)act_dtype, A, weights, row_of, T, H, top_k, dy, dweights, device_status,
                     (int)dy_dtype};
  const bool vec = H % 8 == 0 && aligned16(d_out) && (!dy || aligned16(dy)) && (!dweights || aligned16(y));
  if (vec)
    combine_bwd_kernel<true><<<(unsigned)T, kCombThreads, 0, as_stream(stream)>>>(p);
  else
    combine_bwd_kernel<false><<<(unsigned)T, kCombThreads, 0, as_stream(stream)>>>(p);
  return check_launch("moe_combine_backward");
}

extern "C" moe_status moe_combine_backward(const void *d_out, const void *y, moe_dtype act_dtype, int64_t A,
                                           const float *weights, const int32_t *row_of, int64_t T, int64_t H,
                                           int32_t top_k, void *dy, float *dweights, int32_t *device_status,
                                           void *stream) {
  return moe_combine_backward_dt(d_out, y, act_dtype, A, weights, row_of, T, H, top_k, dy, act_dtype, dweights,
                                 device_status, stream);
}

extern "C" moe_status moe_swiglu_backward_dt(const void *dh, const void *G, const void *U, moe_dtype act_dtype,
                                             int64_t A, int64_t I, void *dG, void *dU, moe_dtype grad_dtype,
                                             int32_t *device_status, void *stream) {
  if (A < 0 || I < 1) return set_error(MOE_ERR_INVALID_ARGUMENT, "moe_swiglu_backward: bad sizes");
  if (act_dtype != MOE_F16 && act_dtype != MOE_BF16)
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "moe_swiglu_backward: act_dtype must be F16 or BF16");
  if (grad_dtype != MOE_F16 && grad_dtype != MOE_BF16)
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "moe_swiglu_backward: grad_dtype must be F16 or BF16");
  if (A == 0) return MOE_OK;
  if (!dh || !G || !U || !dG || !dU) return set_error(MOE_ERR_INVALID_ARGUMENT, "moe_swiglu_backward: NULL pointer");
  SwigluBwdParams p{static_cast<const uint16_t *>(dh), static_cast<const uint16_t *>(G),
                    static_cast<const uint16_t *>(U), static_cast<uint16_t *>(dG), static_cast<uint16_t *>(dU),
                    (int)act_dtype, A * I, 0, (int)grad_dtype, device_status};
  p.vec = aligned16(dh) && aligned16(G) && aligned16(U) && aligned16(dG) && aligned16(dU);
  int64_t blocks = (p.n / (p.vec ? 8 : 1) + 255) / 256;
  int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  swiglu_bwd_kernel<<<(unsigned)blocks, 256, 0, as_stream(stream)>>>(p);
  return check_launch("moe_swiglu_backward");
}

extern "C" moe_status moe_swiglu_backward(const void *dh, const void *G, const void *U, moe_dtype act_dtype,
                                          int64_t A, int64_t I, void *dG, void *dU, void *stream) {
  return moe_swiglu_backward_dt(dh, G, U, act_dtype, A, I, dG, dU, act_dtype, nullptr, stream);
}
