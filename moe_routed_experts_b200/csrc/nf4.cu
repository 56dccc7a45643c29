// Grouped projections with NF4 payloads: ruda-tensor 0.21.34,
// src/packed_experts.rs, PackedExpertPayload::Nf4 ("original RUDA
// high-nibble-first flat-block NF4"; packed scales and codebook frozen; any
// of gate/up/down may use it independently of the others).  The pages print
// no layout; the reading is the 4-bit NormalFloat data type of QLoRA
// (Dettmers et al., 2023): codes uint8 [E, K*N/2] over the logical [K, N]
// matrix flattened row-major (flat element f = kk*N + n in byte f/2, the high
// nibble when f is even), one F32 absmax scale per `block` consecutive
// elements, a 16-entry F32 codebook, and the coefficient
//   W[kk, n] = RNE_cdt(codebook[q] * absmax)   (the F32 x F32 product exact,
//   rounded once to the coefficient dtype, F16 or BF16).
//
// Warp-level tensor-core tiles (mma.sync m16n8k16, FP32 accumulate): each
// warp dequantizes a 16 x 64 coefficient tile into its own shared-memory
// slot (one 16-byte load of codes per lane; codebook entries from a lane
// shuffle; the product in FP64, then one rounding) and reads the MMA
// fragments with ldmatrix (transposed for the forward, where the output
// features are the MMA's M).  CTA = (64 output columns, one expert) for the
// forward, (64 input rows, one expert) for the input VJP; 4 warps split the
// reduction and sum in shared memory in a fixed order.
#include "proj.cuh"
#include "tma.cuh"

namespace moe {

namespace nf4 {
constexpr int kPitch = 72;  // b16 elements per tile row (64 + 8: conflict-free ldmatrix rows)
}

struct Nf4Params {
  const uint16_t *x;  // [A, K] forward input, or [A, N] gradient
  int act_dt;
  int64_t A, K, N;
  const int32_t *offsets;
  int E;
  const uint8_t *codes;    // [E, K*N/2]
  const float *absmax;     // [E, K*N/block]
  const float *codebook;   // [16]
  int64_t block;
  const void *bias;        // [E, N] or NULL (forward)
  int bias_dt;
  uint16_t *out;           // [A, N] (forward) or [A, K] (VJP)
  int32_t *status;
};

template <typename MT>
__device__ __forceinline__ uint16_t rne_from_double(double v) {
  if constexpr (std::is_same<MT, __half>::value) return __half_as_ushort(__double2half(v));
  else return __bfloat16_as_ushort(__double2bfloat16(v));
}

// Coefficients of 32 consecutive flat elements starting at f0 (a multiple of
// 32, inside one block), as 16 packed pairs.  cb: this lane's codebook entry
// (lane & 15).
template <typename MT>
__device__ __forceinline__ void nf4_dequant32(const uint8_t *codes, const float *absmax, int64_t block, int64_t f0,
                                              float cb, uint32_t (&pairs)[16]) {
  const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(codes + f0 / 2));
  const double a = (double)__ldg(absmax + f0 / block);
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t byte = (w[i] >> (8 * b)) & 0xFFu;
      const float hi = __shfl_sync(0xffffffffu, cb, (int)(byte >> 4));   // even element
      const float lo = __shfl_sync(0xffffffffu, cb, (int)(byte & 15u));  // odd element
      const uint16_t e0 = rne_from_double<MT>((double)hi * a), e1 = rne_from_double<MT>((double)lo * a);
      pairs[4 * i + b] = uint32_t(e0) | (uint32_t(e1) << 16);
    }
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr, bool trans) {
  if (trans)
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
  else
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// ------------------------------------------------------------------ forward

template <typename MT>
__global__ void __launch_bounds__(128) nf4_fwd_kernel(Nf4Params p) {
  pdl_enter();  // programmatic dependent launch: the previous kernel is done
  uint32_t act_bad = 0;
  __shared__ __align__(16) uint16_t tile[4][16][nf4::kPitch];  // per warp: [row kk][column n]
  __shared__ float red[4][8][64];
  const int e = blockIdx.y;
  int64_t r0, r1;
  if (!expert_rows(p.offsets, p.E, p.A, e, p.status, r0, r1)) return;
  const int m = (int)(r1 - r0);
  if (m <= 0) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int64_t n0 = (int64_t)blockIdx.x * 64;
  const uint8_t *codes = p.codes + (int64_t)e * (p.K * p.N / 2);
  const float *absmax = p.absmax + (int64_t)e * (p.K * p.N / p.block);
  const float cb = __ldg(p.codebook + (lane & 15));
  const int64_t steps = p.K / 16;
  const uint32_t tbase = smem_u32(&tile[warp][0][0]);
  // ldmatrix.trans addresses: matrix j = lane / 8 holds rows kk = 8 (j >> 1) + lane % 8,
  // columns 8 (j & 1) .. +7 of the 16-column block of m-tile mt
  const int lr = 8 * ((lane >> 3) >> 1) + (lane & 7), lc = 8 * ((lane >> 3) & 1);
  for (int tok0 = 0; tok0 < m; tok0 += 8) {
    float acc[4][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[mt][i] = 0.f;
    const int tr = tok0 + g;
    const bool xok = tr < m;
    const uint16_t *xrow = p.x + (r0 + (xok ? tr : 0)) * p.K;
    for (int64_t s = warp; s < steps; s += 4) {
      // dequantize rows 16 s .. 16 s + 15, columns n0 .. n0 + 63: lane -> row lane / 2, half lane % 2
      {
        const int rr = lane >> 1, hh = lane & 1;
        uint32_t pr[16];
        nf4_dequant32<MT>(codes, absmax, p.block, (16 * s + rr) * p.N + n0 + 32 * hh, cb, pr);
        uint4 *dst = reinterpret_cast<uint4 *>(&tile[warp][rr][32 * hh]);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pr[4 * i], pr[4 * i + 1], pr[4 * i + 2], pr[4 * i + 3]);
      }
      __syncwarp();
      // activations: the MMA's K index 2t, 2t + 1, 2t + 8, 2t + 9 of this step
      uint32_t b0 = 0, b1 = 0;
      if (xok) {
        uint32_t bb[2] = {__ldg(reinterpret_cast<const uint32_t *>(xrow + 16 * s + 2 * t)),
                          __ldg(reinterpret_cast<const uint32_t *>(xrow + 16 * s + 2 * t + 8))};
        act_pairs_to_mt<MT, 2>(bb, p.act_dt, act_bad);
        b0 = bb[0];
        b1 = bb[1];
      }
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        uint32_t a[4];
        ldsm_x4(a, tbase + (uint32_t)((lr * nf4::kPitch + 16 * mt + lc) * 2), true);
        mma16816<MT>(acc[mt], a, b0, b1);
      }
      __syncwarp();
    }
    // acc[mt] = (column 16 mt + g | + 8) x (token 2t | 2t + 1)
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      const int f = 16 * mt + g, tk = 2 * t;
      red[warp][tk][f] = acc[mt][0];
      red[warp][tk + 1][f] = acc[mt][1];
      red[warp][tk][f + 8] = acc[mt][2];
      red[warp][tk + 1][f + 8] = acc[mt][3];
    }
    __syncthreads();
    for (int u = threadIdx.x; u < 8 * 8; u += blockDim.x) {
      const int tk = u >> 3, fq = (u & 7) * 8;
      if (tok0 + tk >= m) continue;
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        float v[2];
#pragma unroll
        for (int d = 0; d < 2; ++d) {
          float sum = red[0][tk][fq + i + d] + red[1][tk][fq + i + d];
          sum += red[2][tk][fq + i + d];
          sum += red[3][tk][fq + i + d];
          if (p.bias) sum += ld_as_float(p.bias, p.bias_dt, (int64_t)e * p.N + n0 + fq + i + d);
          v[d] = sum;
        }
        o[i / 2] = uint32_t(f32_to_bits(v[0], p.act_dt)) | (uint32_t(f32_to_bits(v[1], p.act_dt)) << 16);
      }
      *reinterpret_cast<uint4 *>(p.out + (r0 + tok0 + tk) * p.N + n0 + fq) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __syncthreads();
  }
  if (act_bad) report(p.status, MOE_DEVICE_ERR_ACT_RANGE);
}

// ------------------------------------------------------------------ input VJP
//
// dinput[r, kk] = sum_n grad[r, n] W[kk, n]: the MMA's M = input rows kk (64
// per CTA, four m-tiles), K = output columns n (16 per step), so the
// dequantized tile [kk][n] is the A operand as stored (ldmatrix, no
// transpose).  Lane l dequantizes kk rows 2l and 2l + 1, 32 columns each
// (one 16-byte load of codes per row): a 64 x 32 tile feeds two MMA steps.

template <typename MT>
__global__ void __launch_bounds__(128) nf4_bwd_kernel(Nf4Params p) {
  pdl_enter();  // programmatic dependent launch: the previous kernel is done
  uint32_t act_bad = 0;
  __shared__ __align__(16) uint16_t tile[4][64][40];  // per warp: [row kk][32 columns n] (+8 pad)
  __shared__ float red[4][8][64];
  const int e = blockIdx.y;
  int64_t r0, r1;
  if (!expert_rows(p.offsets, p.E, p.A, e, p.status, r0, r1)) return;
  const int m = (int)(r1 - r0);
  if (m <= 0) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int64_t k0 = (int64_t)blockIdx.x * 64;
  const uint8_t *codes = p.codes + (int64_t)e * (p.K * p.N / 2);
  const float *absmax = p.absmax + (int64_t)e * (p.K * p.N / p.block);
  const float cb = __ldg(p.codebook + (lane & 15));
  const int64_t steps = p.N / 32;  // 32 columns per dequantized tile
  const uint32_t tbase = smem_u32(&tile[warp][0][0]);
  // ldmatrix (no transpose): matrix j = lane / 8: rows 8 (j & 1) + lane % 8, columns 8 (j >> 1) .. +7
  const int lr = 8 * ((lane >> 3) & 1) + (lane & 7), lc = 8 * ((lane >> 3) >> 1);
  for (int tok0 = 0; tok0 < m; tok0 += 8) {
    float acc[4][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[mt][i] = 0.f;
    const int tr = tok0 + g;
    const bool gok = tr < m;
    const uint16_t *grow = p.x + (r0 + (gok ? tr : 0)) * p.N;
    for (int64_t s = warp; s < steps; s += 4) {
      // dequantize rows k0 .. k0 + 63, columns 32 s .. 32 s + 31: lane -> rows 2 lane, 2 lane + 1
#pragma unroll
      for (int d = 0; d < 2; ++d) {
        const int rr = 2 * lane + d;
        uint32_t pr[16];
        nf4_dequant32<MT>(codes, absmax, p.block, (k0 + rr) * p.N + 32 * s, cb, pr);
        uint4 *dst = reinterpret_cast<uint4 *>(&tile[warp][rr][0]);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pr[4 * i], pr[4 * i + 1], pr[4 * i + 2], pr[4 * i + 3]);
      }
      __syncwarp();
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // two 16-column MMA steps of the tile
        uint32_t b0 = 0, b1 = 0;
        if (gok) {
          const int64_t nn = 32 * s + 16 * h + 2 * t;
          uint32_t bb[2] = {__ldg(reinterpret_cast<const uint32_t *>(grow + nn)),
                            __ldg(reinterpret_cast<const uint32_t *>(grow + nn + 8))};
          act_pairs_to_mt<MT, 2>(bb, p.act_dt, act_bad);
          b0 = bb[0];
          b1 = bb[1];
        }
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          uint32_t a[4];
          ldsm_x4(a, tbase + (uint32_t)(((16 * mt + lr) * 40 + 16 * h + lc) * 2), false);
          mma16816<MT>(acc[mt], a, b0, b1);
        }
      }
      __syncwarp();
    }
    // acc[mt] = (input row 16 mt + g | + 8) x (token 2t | 2t + 1)
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      const int rr = 16 * mt + g, tk = 2 * t;
      red[warp][tk][rr] = acc[mt][0];
      red[warp][tk + 1][rr] = acc[mt][1];
      red[warp][tk][rr + 8] = acc[mt][2];
      red[warp][tk + 1][rr + 8] = acc[mt][3];
    }
    __syncthreads();
    for (int u = threadIdx.x; u < 8 * 8; u += blockDim.x) {
      const int tk = u >> 3, rq = (u & 7) * 8;
      if (tok0 + tk >= m) continue;
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        float v[2];
#pragma unroll
        for (int d = 0; d < 2; ++d) {
          float sum = red[0][tk][rq + i + d] + red[1][tk][rq + i + d];
          sum += red[2][tk][rq + i + d];
          sum += red[3][tk][rq + i + d];
          v[d] = sum;
        }
        o[i / 2] = uint32_t(f32_to_bits(v[0], p.act_dt)) | (uint32_t(f32_to_bits(v[1], p.act_dt)) << 16);
      }
      *reinterpret_cast<uint4 *>(p.out + (r0 + tok0 + tk) * p.K + k0 + rq) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __syncthreads();
  }
  if (act_bad) report(p.status, MOE_DEVICE_ERR_ACT_RANGE);
}

// ------------------------------------------------------------------ C ABI

static moe_status nf4_check(const char *fn, int64_t A, int64_t K, int64_t N, int64_t E, int64_t block,
                            moe_dtype act_dt, moe_dtype coef_dt, const void *in, const int32_t *offsets,
                            const uint8_t *codes, const float *absmax, const float *codebook, const void *out) {
  if (act_dt != MOE_F16 && act_dt != MOE_BF16)
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "%s: activations must be F16 or BF16", fn);
  if (coef_dt != MOE_F16 && coef_dt != MOE_BF16)
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "%s: the coefficient dtype must be F16 or BF16", fn);
  if (A < 0 || E < 1 || E > MOE_MAX_EXPERTS || K < 16 || N < 64 || A > INT32_MAX)
    return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: bad sizes A=%lld K=%lld N=%lld E=%lld", fn, (long long)A,
                     (long long)K, (long long)N, (long long)E);
  if (K % 64 != 0 || N % 64 != 0 || block < 32 || block % 32 != 0 || (K * N) % block != 0)
    return set_error(MOE_ERR_INVALID_ARGUMENT,
                     "%s: this library runs K and N multiples of 64 and blocks a multiple of 32 dividing K*N "
                     "(K=%lld N=%lld block=%lld)", fn, (long long)K, (long long)N, (long long)block);
  if (A == 0) return MOE_OK;
  if (!in || !offsets || !codes || !absmax || !codebook || !out)
    return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: NULL tensor pointer", fn);
  if (!aligned16(in) || !aligned16(codes) || !aligned16(out) || (reinterpret_cast<uintptr_t>(absmax) & 3u))
    return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: tensor not aligned (16 bytes; absmax 4)", fn);
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" moe_status nf4_grouped_projection(const void *input, moe_dtype act_dtype, int64_t A, int64_t K, int64_t N,
                                             const int32_t *offsets, int64_t E, const uint8_t *codes,
                                             const float *absmax, const float *codebook, int64_t block,
                                             moe_dtype coef_dtype, const void *bias, moe_dtype bias_dtype,
                                             void *output, int32_t *device_status, void *stream) {
  const char *fn = "nf4_grouped_projection";
  moe_status s = nf4_check(fn, A, K, N, E, block, act_dtype, coef_dtype, input, offsets, codes, absmax, codebook,
                           output);
  if (s != MOE_OK || A == 0) return s;
  if (bias && !valid_dtype(bias_dtype)) return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "%s: bad bias dtype", fn);
  Nf4Params p{static_cast<const uint16_t *>(input), act_dtype, A, K, N, offsets, (int)E, codes, absmax, codebook,
              block, bias, bias_dtype, static_cast<uint16_t *>(output), device_status};
  const dim3 grid((unsigned)(N / 64), (unsigned)E);
  if (coef_dtype == MOE_BF16) launch_pdl(nf4_fwd_kernel<__nv_bfloat16>, grid, dim3(128), 0, as_stream(stream), p);
  else launch_pdl(nf4_fwd_kernel<__half>, grid, dim3(128), 0, as_stream(stream), p);
  return check_launch(fn);
}

extern "C" moe_status nf4_input_backward(const void *grad, moe_dtype grad_dtype, int64_t A, int64_t N, int64_t K,
                                         const int32_t *offsets, int64_t E, const uint8_t *codes,
                                         const float *absmax, const float *codebook, int64_t block,
                                         moe_dtype coef_dtype, void *dinput, int32_t *device_status, void *stream) {
  const char *fn = "nf4_input_backward";
  moe_status s = nf4_check(fn, A, K, N, E, block, grad_dtype, coef_dtype, grad, offsets, codes, absmax, codebook,
                           dinput);
  if (s != MOE_OK || A == 0) return s;
  Nf4Params p{static_cast<const uint16_t *>(grad), grad_dtype, A, K, N, offsets, (int)E, codes, absmax, codebook,
              block, nullptr, MOE_F32, static_cast<uint16_t *>(dinput), device_status};
  const dim3 grid((unsigned)(K / 64), (unsigned)E);
  if (coef_dtype == MOE_BF16) launch_pdl(nf4_bwd_kernel<__nv_bfloat16>, grid, dim3(128), 0, as_stream(stream), p);
  else launch_pdl(nf4_bwd_kernel<__half>, grid, dim3(128), 0, as_stream(stream), p);
  return check_launch(fn);
}
