// Grouped AWQ projections on warp-level tensor-core tiles (mma.sync
// m16n8k16, FP32 accumulate): the path for small per-expert batches
// (decode), where the packed-weight bytes bound the time.
//
// ruda-tensor 0.21.34, src/packed_experts.rs -- FrozenPackedExpertOps
//   (packed_expert_forward / packed_swiglu_forward / the input VJPs);
// ruda-tensor 0.21.33, src/frozen_awq.rs -- FrozenAwqOps (AWQ nibble order
//   and scale-dtype coefficient rounding kept; the input VJP applies the
//   transpose of the same rounded coefficients).
//
// Forward tile (weights as the MMA's A operand, tokens as B):
//   CTA = (64 output features = 8 packed word columns, one expert), 4 warps
//   splitting the K loop; partial sums are reduced in shared memory in a
//   fixed warp order.  Lane (g, t) owns word column g of the slab and, per
//   16-row K step, the words of rows 4t..4t+3.  A-fragment row g is the
//   feature in nibble slot p, row g+8 the one in slot p+4 (logical columns
//   2p and 2p+1 of the word); the MMA's K index k maps to input row
//   {2t,2t+1,2t+8,2t+9} -> {4t,4t+1,4t+2,4t+3}, so two words of rows 4t and
//   4t+1 interleaved by PRMT give the A pair registers directly.  The token
//   B fragment is then 4 consecutive activations of one row (one 8-byte
//   load).  Coefficients are formed in registers and never stored.
//
// Input-VJP tile (weights as A again, but A rows = input rows kk and the
//   MMA's K = output features): one word gives (slot p, slot p+4) = logical
//   columns (2p, 2p+1) at the same row, which is an A pair as it stands.
//   CTA = (64 input rows, one expert), 4 warps splitting the feature range.
#include "dequant.cuh"
#include "proj.cuh"

namespace moe {

// ------------------------------------------------------------------ forward

template <typename MT, int NPROJ, int NT>
__global__ void __launch_bounds__(128) awq_fwd_mma_kernel(ProjParams p) {
  pdl_enter();  // programmatic dependent launch: the previous kernel is done
  uint32_t act_bad = 0;  // a converted input outside F16's normal range
  constexpr int D = 2;  // K steps of loads in flight per warp
  __shared__ float red[4][NPROJ][8 * NT][64];
  const int e = blockIdx.y;
  int64_t r0, r1;
  if (!expert_rows(p.offsets, p.E, p.A, e, p.status, r0, r1)) return;
  const int m = (int)(r1 - r0);
  if (m <= 0) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int64_t NW = p.N / 8;
  const int64_t wc = (int64_t)blockIdx.x * 8 + g;
  const bool wc_ok = wc < NW;
  const int64_t wcs = wc_ok ? wc : 0;
  const int64_t steps = p.K / 16;
  const int64_t s_begin = steps * warp / 4, s_end = steps * (warp + 1) / 4;
  const int64_t ngroups = p.K / p.group;
  const int32_t *qwp[NPROJ];
  const int32_t *qzp[NPROJ];
  const uint16_t *scp[NPROJ];
#pragma unroll
  for (int j = 0; j < NPROJ; ++j) {
    qwp[j] = p.qw[j] + (int64_t)e * p.K * NW + wcs + (int64_t)(4 * t) * NW;
    qzp[j] = p.qz[j] + (int64_t)e * ngroups * NW + wcs;
    scp[j] = p.sc[j] + (int64_t)e * ngroups * p.N + 8 * wcs;
  }

  for (int tok0 = 0; tok0 < m; tok0 += 8 * NT) {
    float acc[NPROJ][NT][4][4];
#pragma unroll
    for (int j = 0; j < NPROJ; ++j)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[j][nt][q][i] = 0.f;
    const uint16_t *xrow[NT];
    bool xok[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int tr = tok0 + nt * 8 + g;
      xok[nt] = tr < m;
      xrow[nt] = p.x + act_row(p, r0 + (xok[nt] ? tr : 0)) * p.K + 4 * t;
    }
    FwdConsts<MT> cst[NPROJ];
    int64_t cur_grp = -1;
    uint32_t wbuf[D][NPROJ][4];
    uint2 xbuf[D][NT];
#pragma unroll
    for (int d = 0; d < D; ++d) {
      const int64_t s = s_begin + d;
      if (s < s_end) {
#pragma unroll
        for (int j = 0; j < NPROJ; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i) wbuf[d][j][i] = wc_ok ? ldg_nc_u32(qwp[j] + (s * 16 + i) * NW) : 0u;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          xbuf[d][nt] = xok[nt] ? __ldg(reinterpret_cast<const uint2 *>(xrow[nt] + s * 16)) : make_uint2(0, 0);
      }
    }
    for (int64_t base = s_begin; base < s_end; base += D) {
#pragma unroll
      for (int d = 0; d < D; ++d) {
        const int64_t s = base + d;
        if (s < s_end) {
          const int64_t grp = (int64_t)((uint32_t)(s * 16) / (uint32_t)p.group);
          if (grp != cur_grp) {
            cur_grp = grp;
#pragma unroll
            for (int j = 0; j < NPROJ; ++j) {
              const uint32_t zw = wc_ok ? (uint32_t)__ldg(qzp[j] + grp * NW) : 0u;
              const uint4 sv = wc_ok ? ldg16(scp[j] + grp * p.N) : make_uint4(0, 0, 0, 0);
              cst[j].load(zw, sv);
            }
          }
          uint32_t b0[NT], b1[NT];
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            uint32_t bb[2] = {xbuf[d][nt].x, xbuf[d][nt].y};
            act_pairs_to_mt<MT, 2>(bb, p.act_dt, act_bad);
            b0[nt] = bb[0];
            b1[nt] = bb[1];
          }
#pragma unroll
          for (int j = 0; j < NPROJ; ++j) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t a[4];
              fwd_pairs<MT>(wbuf[d][j][0], wbuf[d][j][1], q, cst[j], a[0], a[1]);
              fwd_pairs<MT>(wbuf[d][j][2], wbuf[d][j][3], q, cst[j], a[2], a[3]);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) mma16816<MT>(acc[j][nt][q], a, b0[nt], b1[nt]);
            }
          }
          const int64_t sn = s + D;
          if (sn < s_end) {
#pragma unroll
            for (int j = 0; j < NPROJ; ++j)
#pragma unroll
              for (int i = 0; i < 4; ++i) wbuf[d][j][i] = wc_ok ? ldg_nc_u32(qwp[j] + (sn * 16 + i) * NW) : 0u;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              xbuf[d][nt] = xok[nt] ? __ldg(reinterpret_cast<const uint2 *>(xrow[nt] + sn * 16)) : make_uint2(0, 0);
          }
        }
      }
    }
    // partial sums -> shared memory: acc[j][nt][q] = (feature 8g+2q | 8g+2q+1) x (token 2t | 2t+1)
#pragma unroll
    for (int j = 0; j < NPROJ; ++j)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int f = 8 * g + 2 * q, tk = nt * 8 + 2 * t;
          red[warp][j][tk][f] = acc[j][nt][q][0];
          red[warp][j][tk + 1][f] = acc[j][nt][q][1];
          red[warp][j][tk][f + 1] = acc[j][nt][q][2];
          red[warp][j][tk + 1][f + 1] = acc[j][nt][q][3];
        }
    __syncthreads();
    // epilogue: one (token, 8 features) unit per thread and pass
    for (int u = threadIdx.x; u < 8 * NT * 8; u += blockDim.x) {
      const int tk = u >> 3, fq = (u & 7) * 8;
      const int64_t n0 = (int64_t)blockIdx.x * 64 + fq;
      if (tok0 + tk >= m || n0 >= p.N) continue;
      const int64_t row = r0 + tok0 + tk;
      float v[NPROJ][8];
#pragma unroll
      for (int j = 0; j < NPROJ; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float s = red[0][j][tk][fq + i] + red[1][j][tk][fq + i];
          s += red[2][j][tk][fq + i];
          s += red[3][j][tk][fq + i];
          if (p.bias[j]) s += ld_as_float(p.bias[j], p.bias_dt, (int64_t)e * p.N + n0 + i);
          v[j][i] = s;
        }
      uint32_t o[4];
      if (NPROJ == 2) {
        uint32_t og[4], ou[4];
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          const uint16_t gb0 = f32_to_bits(v[0][i], p.odt), gb1 = f32_to_bits(v[0][i + 1], p.odt);
          const uint16_t ub0 = f32_to_bits(v[NPROJ - 1][i], p.odt), ub1 = f32_to_bits(v[NPROJ - 1][i + 1], p.odt);
          const float g0 = bits_to_f32(gb0, p.odt), g1 = bits_to_f32(gb1, p.odt);
          const float u0 = bits_to_f32(ub0, p.odt), u1 = bits_to_f32(ub1, p.odt);
          const float h0 = g0 / (1.f + expf(-g0)) * u0, h1 = g1 / (1.f + expf(-g1)) * u1;
          og[i / 2] = uint32_t(gb0) | (uint32_t(gb1) << 16);
          ou[i / 2] = uint32_t(ub0) | (uint32_t(ub1) << 16);
          o[i / 2] = round_h(p, h0, h1, p.odt == MOE_BF16);
        }
        if (p.gout) *reinterpret_cast<uint4 *>(p.gout + row * p.N + n0) = make_uint4(og[0], og[1], og[2], og[3]);
        if (p.uout) *reinterpret_cast<uint4 *>(p.uout + row * p.N + n0) = make_uint4(ou[0], ou[1], ou[2], ou[3]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; i += 2)
          o[i / 2] = uint32_t(f32_to_bits(v[0][i], p.odt)) | (uint32_t(f32_to_bits(v[0][i + 1], p.odt)) << 16);
      }
      *reinterpret_cast<uint4 *>(p.out + row * p.N + n0) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __syncthreads();
  }
  if (act_bad) report(p.status, MOE_DEVICE_ERR_ACT_RANGE);
}

// ------------------------------------------------------------------ input VJP

template <typename MT, int NPROJ, int NT>
__global__ void __launch_bounds__(128) awq_bwd_mma_kernel(BwdParams p) {
  uint32_t act_bad = 0;  // a converted input outside F16's normal range
  __shared__ float red[4][8 * NT][64];
  const int e = blockIdx.y;
  int64_t r0, r1;
  if (!expert_rows(p.offsets, p.E, p.A, e, p.status, r0, r1)) return;
  const int m = (int)(r1 - r0);
  if (m <= 0) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int64_t NW = p.N / 8;
  const int64_t kb = (int64_t)blockIdx.x * 64;
  const int64_t ngroups = p.K / p.group;
  const int64_t spp = (NW + 3) / 4;  // K steps (4 word columns) per projection
  const int64_t steps = spp * NPROJ;
  const int64_t s_begin = steps * warp / 4, s_end = steps * (warp + 1) / 4;
  bool mt_ok[4];
  int64_t grp_mt[4];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
    mt_ok[mt] = kb + 16 * mt < p.K;
    grp_mt[mt] = mt_ok[mt] ? (kb + 16 * mt) / p.group : 0;
  }

  for (int tok0 = 0; tok0 < m; tok0 += 8 * NT) {
    float acc[4][NT][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.f;
    int64_t grow[NT];
    bool gok[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int tr = tok0 + nt * 8 + g;
      gok[nt] = tr < m;
      grow[nt] = (r0 + (gok[nt] ? tr : 0)) * p.N;
    }
    int j = (int)(s_begin / spp);
    int64_t sj = s_begin - (int64_t)j * spp;  // step within projection j
    for (int64_t s = s_begin; s < s_end; ++s, ++sj) {
      if (sj == spp) {
        sj = 0;
        ++j;
      }
      const int64_t wc = sj * 4 + t;
      const bool wc_ok = wc < NW;
      const int64_t wcs = wc_ok ? wc : 0;
      const int32_t *qw = p.qw[j] + (int64_t)e * p.K * NW + wcs;
      const int32_t *qz = p.qz[j] + (int64_t)e * ngroups * NW + wcs;
      const uint16_t *sc = p.sc[j] + (int64_t)e * ngroups * p.N + 8 * wcs;
      uint32_t wa[4], wb[4], zw[4];
      uint4 sv[4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        const bool ok = wc_ok && mt_ok[mt];
        const int64_t ka = kb + 16 * mt + g;
        wa[mt] = ok ? ldg_nc_u32(qw + ka * NW) : 0u;
        wb[mt] = ok ? ldg_nc_u32(qw + (ka + 8) * NW) : 0u;
        zw[mt] = ok ? (uint32_t)__ldg(qz + grp_mt[mt] * NW) : 0u;
        sv[mt] = ok ? ldg16(sc + grp_mt[mt] * p.N) : make_uint4(0, 0, 0, 0);
      }
      uint4 gv[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        gv[nt] = (gok[nt] && wc_ok) ? ldg16(p.grad[j] + grow[nt] + 8 * wc) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        uint32_t b0[NT], b1[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          uint32_t bb[2] = {q == 0 ? gv[nt].x : gv[nt].z, q == 0 ? gv[nt].y : gv[nt].w};
          act_pairs_to_mt<MT, 2>(bb, p.gdt, act_bad);
          b0[nt] = bb[0];
          b1[nt] = bb[1];
        }
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          const uint32_t s_lo = q == 0 ? sv[mt].x : sv[mt].z;  // (s[4q], s[4q+1])
          const uint32_t s_hi = q == 0 ? sv[mt].y : sv[mt].w;  // (s[4q+2], s[4q+3])
          uint32_t a[4];
          a[0] = word_pair<MT>(wa[mt], zw[mt], s_lo, 2 * q);
          a[1] = word_pair<MT>(wb[mt], zw[mt], s_lo, 2 * q);
          a[2] = word_pair<MT>(wa[mt], zw[mt], s_hi, 2 * q + 1);
          a[3] = word_pair<MT>(wb[mt], zw[mt], s_hi, 2 * q + 1);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma16816<MT>(acc[mt][nt], a, b0[nt], b1[nt]);
        }
      }
    }
    // acc[mt][nt] = (row 16mt+g | 16mt+g+8) x (token 2t | 2t+1)
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int rr = 16 * mt + g, tk = nt * 8 + 2 * t;
        red[warp][tk][rr] = acc[mt][nt][0];
        red[warp][tk + 1][rr] = acc[mt][nt][1];
        red[warp][tk][rr + 8] = acc[mt][nt][2];
        red[warp][tk + 1][rr + 8] = acc[mt][nt][3];
      }
    __syncthreads();
    for (int u = threadIdx.x; u < 8 * NT * 8; u += blockDim.x) {
      const int tk = u >> 3, rq = (u & 7) * 8;
      const int64_t k0 = kb + rq;
      if (tok0 + tk >= m || k0 >= p.K) continue;
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        float s0 = red[0][tk][rq + i] + red[1][tk][rq + i];
        s0 += red[2][tk][rq + i];
        s0 += red[3][tk][rq + i];
        float s1 = red[0][tk][rq + i + 1] + red[1][tk][rq + i + 1];
        s1 += red[2][tk][rq + i + 1];
        s1 += red[3][tk][rq + i + 1];
        o[i / 2] = uint32_t(f32_to_bits(s0, p.odt)) | (uint32_t(f32_to_bits(s1, p.odt)) << 16);
      }
      *reinterpret_cast<uint4 *>(p.out + (r0 + tok0 + tk) * p.K + k0) = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __syncthreads();
  }
  if (act_bad) report(p.status, MOE_DEVICE_ERR_ACT_RANGE);
}

// ------------------------------------------------------------------ coefficient dump

// mode 0: through the forward PRMT extraction (rows 2i, 2i+1 of a column);
// mode 1: through the input-VJP word extraction.
template <typename MT>
__global__ void awq_dump_kernel(const int32_t *qw, const int32_t *qz, const uint16_t *sc, int64_t K, int64_t N,
                                int group, uint16_t *out, int mode) {
  const int64_t NW = N / 8;
  const int64_t rows = mode == 0 ? K / 2 : K;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < rows * NW;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t w = u % NW, r = u / NW;
    if (mode == 0) {
      const int64_t kk = 2 * r, grp = kk / group;
      FwdConsts<MT> c;
      c.load((uint32_t)qz[grp * NW + w], *reinterpret_cast<const uint4 *>(sc + grp * N + 8 * w));
      const uint32_t wa = (uint32_t)qw[kk * NW + w], wb = (uint32_t)qw[(kk + 1) * NW + w];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t lo, hi;
        fwd_pairs<MT>(wa, wb, q, c, lo, hi);
        out[kk * N + 8 * w + 2 * q] = uint16_t(lo & 0xFFFF);
        out[(kk + 1) * N + 8 * w + 2 * q] = uint16_t(lo >> 16);
        out[kk * N + 8 * w + 2 * q + 1] = uint16_t(hi & 0xFFFF);
        out[(kk + 1) * N + 8 * w + 2 * q + 1] = uint16_t(hi >> 16);
      }
    } else {
      const int64_t kk = r, grp = kk / group;
      const uint32_t zw = (uint32_t)qz[grp * NW + w];
      const uint4 sv = *reinterpret_cast<const uint4 *>(sc + grp * N + 8 * w);
      const uint32_t sp[4] = {sv.x, sv.y, sv.z, sv.w};
      const uint32_t wd = (uint32_t)qw[kk * NW + w];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t c = word_pair<MT>(wd, zw, sp[q], q);
        out[kk * N + 8 * w + 2 * q] = uint16_t(c & 0xFFFF);
        out[kk * N + 8 * w + 2 * q + 1] = uint16_t(c >> 16);
      }
    }
  }
}

// ------------------------------------------------------------------ launchers

template <typename MT, int NPROJ>
static void launch_fwd_t(const ProjParams &p, int nt, cudaStream_t st) {
  dim3 grid((unsigned)((p.N / 8 + 7) / 8), (unsigned)p.E);
  if (nt == 2)
    launch_pdl(awq_fwd_mma_kernel<MT, NPROJ, 2>, grid, dim3(128), 0, st, p);
  else
    launch_pdl(awq_fwd_mma_kernel<MT, NPROJ, 1>, grid, dim3(128), 0, st, p);
}

void launch_fwd_mma(const ProjParams &p, int nproj, bool bf16_mma, int nt, cudaStream_t st) {
  if (bf16_mma) {
    if (nproj == 2) launch_fwd_t<__nv_bfloat16, 2>(p, nt, st);
    else launch_fwd_t<__nv_bfloat16, 1>(p, nt, st);
  } else {
    if (nproj == 2) launch_fwd_t<__half, 2>(p, nt, st);
    else launch_fwd_t<__half, 1>(p, nt, st);
  }
}

template <typename MT, int NPROJ>
static void launch_bwd_t(const BwdParams &p, int nt, cudaStream_t st) {
  dim3 grid((unsigned)((p.K + 63) / 64), (unsigned)p.E);
  if (nt == 2)
    awq_bwd_mma_kernel<MT, NPROJ, 2><<<grid, 128, 0, st>>>(p);
  else
    awq_bwd_mma_kernel<MT, NPROJ, 1><<<grid, 128, 0, st>>>(p);
}

void launch_bwd_mma(const BwdParams &p, int nproj, bool bf16_mma, int nt, cudaStream_t st) {
  if (bf16_mma) {
    if (nproj == 2) launch_bwd_t<__nv_bfloat16, 2>(p, nt, st);
    else launch_bwd_t<__nv_bfloat16, 1>(p, nt, st);
  } else {
    if (nproj == 2) launch_bwd_t<__half, 2>(p, nt, st);
    else launch_bwd_t<__half, 1>(p, nt, st);
  }
}

void launch_dump(const int32_t *qw, const int32_t *qz, const uint16_t *sc, int64_t K, int64_t N, int group,
                 uint16_t *out, int mode, bool bf16_mma, cudaStream_t st) {
  int64_t rows = mode == 0 ? K / 2 : K;
  int64_t units = rows * (N / 8);
  int64_t blocks = (units + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  if (blocks < 1) blocks = 1;
  if (bf16_mma)
    awq_dump_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(qw, qz, sc, K, N, group, out, mode);
  else
    awq_dump_kernel<__half><<<(unsigned)blocks, 256, 0, st>>>(qw, qz, sc, K, N, group, out, mode);
}

}  // namespace moe
