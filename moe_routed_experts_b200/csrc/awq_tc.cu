// Grouped AWQ projections on tcgen05 tensor cores with TMEM accumulators,
// for per-expert batches large enough to fill 128-row tiles (prefill).
//
// ruda-tensor 0.21.34, src/packed_experts.rs -- packed_expert_forward /
//   packed_swiglu_forward (gate/up/down of the selected experts, SwiGLU);
// ruda-tensor 0.21.33, src/frozen_awq.rs -- AWQ nibble order and scale-dtype
//   coefficient rounding; the tensor-core products run in the scale dtype.
//
// Tile: 128 expert rows x 256 output columns (for the gate/up pair: 128
// features of each projection, so SwiGLU sees G and U of a feature in the
// same thread), K in steps of 64.  Persistent CTAs walk the tile list
// (expert-major, row tile, column tile) round-robin.  Warp roles:
//   warp 0  producer: TMA of the activation tile (128 x 64, 128-byte
//           swizzle, K-major) and of the packed words of the step
//           (64 rows x 32 words) into a 3-stage ring;
//   warp 1  allocates 512 TMEM columns (two accumulators); lane 0 issues tcgen05.mma
//           (M=128, N=256, K=16, FP32 accumulate in TMEM) and commits each
//           stage back to the producer and the finished tile to the epilogue;
//   warps 2-9 dequantize: each thread forms the coefficients of 8 packed
//           words (8 features at one input row each, in logical order) and
//           stores them as 16-byte chunks of the B operand, laid out MN-major
//           with 128-byte swizzle (8-row x 64-column atoms); when the
//           activations are not in the scale dtype they also convert the
//           activation tile in place;
//   warps 10-17 (two per TMEM lane quarter, one per column half) read a
//           finished accumulator (tcgen05.ld 32x32b), add the bias, round,
//           apply SwiGLU and store, while the tensor core fills the other of
//           the two TMEM buffers.
// Coefficients are exact per the operation: RNE_scale((q - z) s) formed with
// the magic-number conversion (see common.cuh), never written to HBM.
#include <cudaTypedefs.h>

#include "dequant.cuh"
#include "proj.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace moe {

namespace tc {
constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kLStages = 6;  // TMA ring: activation tile + packed words, six deep to cover the load latency
constexpr int kBStages = 2;  // coefficient ring
constexpr int kDqWarps = 8;
constexpr int kEpWarps = 8;                                // two per TMEM lane quarter (column halves)
constexpr int kThreads = (2 + kDqWarps + kEpWarps) * 32;  // 576
constexpr int kABytes = kBM * kBK * 2;          // 16 KB activation tile
constexpr int kBBytes = kBN * kBK * 2;          // 32 KB coefficient tile
constexpr int kPBytes = kBK * (kBN / 8) * 4;    // 8 KB packed words
constexpr int kLBytes = kABytes + kPBytes;    // one TMA stage (24 KB: 1 KB aligned)
constexpr int kTmemCols = 512;  // two 128 x 256 FP32 accumulators
}  // namespace tc

// ------------------------------------------------------------------ kernel

struct TileInfo {
  int e, mt, nt;
  int64_t r0;  // first row of the expert
  int m;       // rows of the expert
};

template <typename MT, int NPROJ>
__global__ void __launch_bounds__(tc::kThreads, 1)
    awq_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w0,
                      const __grid_constant__ CUtensorMap map_w1, ProjParams p) {
  pdl_enter();  // programmatic dependent launch: the previous kernel is done
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t *lring = smem;                           // kLStages x [A | packed]
  uint8_t *bring = smem + kLStages * kLBytes;      // kBStages x B
  uint64_t *full = reinterpret_cast<uint64_t *>(bring + kBStages * kBBytes);
  uint64_t *empty = full + kLStages;               // MMA commit (A read) + dequant warps (words read)
  uint64_t *bready = empty + kLStages;
  uint64_t *bfree = bready + kBStages;
  uint64_t *accfull = bfree + kBStages;  // [2]
  uint64_t *accempty = accfull + 2;     // [2]
  uint64_t *drain = accempty + 2;       // the issuer's last commit: no MMA in flight at teardown
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int32_t *abort = reinterpret_cast<volatile int32_t *>(tmem_slot + 1);
  float *bias_s = reinterpret_cast<float *>(tmem_slot + 4);  // [2 tiles][256]: the tile's bias, staged
  int32_t *pre = reinterpret_cast<int32_t *>(bias_s + 2 * kBN);  // [E + 1]
  int32_t *cnt = pre + (p.E + 1);                             // [E]
  int32_t *tmp = cnt + p.E;                                   // [32]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;
  const int64_t K = p.K, NW = p.N / 8;
  const int feat_tile = NPROJ == 2 ? kBN / 2 : kBN;          // output features per tile
  const int NT = (int)((p.N + feat_tile - 1) / feat_tile);  // column tiles per row tile
  const int nk = (int)(K / kBK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLStages; ++s) {
      mbar_init(&full[s], p.gather ? 1 + 32 : 1);  // + the producer lanes' gathered rows
      mbar_init(&empty[s], 1 + kDqWarps);
    }
    for (int b = 0; b < kBStages; ++b) {
      mbar_init(&bready[b], kDqWarps);
      mbar_init(&bfree[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], kEpWarps);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int32_t a = p.offsets[e], b = p.offsets[e + 1];
    const bool bad = a < 0 || b < a || (int64_t)b > p.A || (e == 0 && a != 0) || (e == E - 1 && (int64_t)b != p.A);
    if (bad && blockIdx.x == 0) report(p.status, MOE_DEVICE_ERR_OFFSETS);
    cnt[e] = bad ? 0 : NT * ((b - a + kBM - 1) / kBM);
  }
  __syncthreads();
  block_exclusive_scan(cnt, E, pre, tmp);
  const int64_t total = pre[E];
  if ((int64_t)blockIdx.x >= total) return;  // no tile for this CTA (uniform)

  auto tile_info = [&](int64_t tile) {
    TileInfo ti;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= tile) lo = mid;
      else hi = mid - 1;
    }
    ti.e = lo;
    const int64_t local = tile - pre[lo];
    ti.mt = (int)(local / NT);
    ti.nt = (int)(local % NT);
    ti.r0 = p.offsets[lo];
    ti.m = p.offsets[lo + 1] - (int32_t)ti.r0;
    return ti;
  };

  if (warp == 1) {  // TMEM allocation (whole warp)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer (lane 0, by TMA).  With a gather, every lane
    // copies four rows of each activation step with 16-byte cp.async into
    // the swizzled atom (lane L: tile rows L, L + 32, L + 64, L + 96) and
    // arrives on the stage's full barrier once its copies of that stage
    // landed (one stage behind, so two stages stay in flight), after a proxy
    // fence for the tensor core.
    const bool gather = p.gather != nullptr;
    if (gather || lane == 0) {
      const uint32_t rowoff = (uint32_t)((lane >> 3) * 1024 + (lane & 7) * 128);
      uint32_t it = 0;  // stages issued
      bool live = true;
      bool pend = false;  // gather: a stage whose rows this lane still has to deliver
      uint32_t pend_s = 0;
      auto deliver = [&](bool all) {
        if (!pend) return;
        if (all) cp_async_wait<0>();
        else cp_async_wait<1>();
        fence_proxy_async_smem();
        mbar_arrive(&full[pend_s]);
        pend = false;
      };
      for (int64_t tile = blockIdx.x; tile < total && live; tile += gridDim.x) {
        const TileInfo ti = tile_info(tile);
        const int32_t row0 = (int32_t)(ti.r0 + (int64_t)ti.mt * kBM);
        const uint16_t *srow[4] = {p.x, p.x, p.x, p.x};  // gather: x rows of tile rows lane + 32 i
        if (gather) {
#pragma unroll
          for (int i = 0; i < 4; ++i) srow[i] = p.x + act_row(p, min((int64_t)row0 + lane + 32 * i, p.A - 1)) * K;
        }
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t s = it % kLStages, use = it / kLStages;
          bool ok = true;
          uint8_t *st = lring + s * kLBytes;
          if (lane == 0) {
            ok = use == 0 || tc_wait(&empty[s], (use - 1) & 1, p.status, abort);
            if (ok) mbar_arrive_expect_tx(&full[s], gather ? kPBytes : kLBytes);
          }
          if (gather) ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) {
            live = false;
            break;
          }
          if (gather) {
            const uint32_t sbase = smem_u32(st) + rowoff;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint16_t *src = srow[i] + (int64_t)kb * kBK;
#pragma unroll
              for (int cc = 0; cc < 8; ++cc) cp_async16(sbase + i * 4096 + ((cc ^ (lane & 7)) << 4), src + cc * 8);
            }
            cp_async_commit();
            deliver(false);  // the previous stage (at most this one's copies left in flight)
            pend = true;
            pend_s = s;
          }
          if (lane == 0) {
            if (!gather) tma_load_2d(st, &map_x, &full[s], kb * kBK, row0);
            const int32_t wrow = (int32_t)(ti.e * K + (int64_t)kb * kBK);
            if (NPROJ == 2) {
              tma_load_2d(st + kABytes, &map_w0, &full[s], ti.nt * 16, wrow);
              tma_load_2d(st + kABytes + kPBytes / 2, &map_w1, &full[s], ti.nt * 16, wrow);
            } else {
              tma_load_2d(st + kABytes, &map_w0, &full[s], ti.nt * 32, wrow);
            }
          }
        }
      }
      if (gather) deliver(true);  // every issued stage complete before the drain below
      if (lane == 0) tma_drain(full, it, kLStages, p.status);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: tile t accumulates in TMEM buffer t & 1
    if (lane == 0) {
      constexpr uint32_t fmt = std::is_same<MT, __half>::value ? 0u : 1u;
      // D F32, A/B in the scale dtype, A K-major, B MN-major, N = 256, M = 128
      const uint32_t idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | (1u << 16) | ((uint32_t)(kBN >> 3) << 17) |
                             ((uint32_t)(kBM >> 4) << 24);
      uint32_t it = 0, tcount = 0;
      bool live = true;
      for (int64_t tile = blockIdx.x; tile < total; tile += gridDim.x, ++tcount) {
        const uint32_t buf = tcount & 1, use = tcount >> 1;
        if (use > 0 && !tc_wait(&accempty[buf], (use - 1) & 1, p.status, abort)) break;
        tc_fence_after();
        const uint32_t dacc = tmem + buf * kBN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t s = it % kLStages, b = it % kBStages;
          // the dequant warps arrive on bready only after the stage's TMA landed
          if (!tc_wait(&bready[b], (it / kBStages) & 1, p.status, abort)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(lring + s * kLBytes);
          const uint32_t b_addr = smem_u32(bring + b * kBBytes);
          const uint64_t adesc = smem_desc(a_addr, 16, 1024);    // K-major, 8-row groups 1 KB apart
          const uint64_t bdesc = smem_desc(b_addr, 8192, 1024);  // MN-major: 64-col groups 8 KB, 8-row groups 1 KB
#pragma unroll
          for (int j = 0; j < kBK / 16; ++j)
            umma_f16(dacc, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(128 * j), idesc, (kb | j) != 0);
          umma_commit(&empty[s]);
          umma_commit(&bfree[b]);
        }
        if (!live) break;
        umma_commit(&accfull[buf]);
      }
      umma_commit(drain);  // arrives once every MMA issued above has completed
      mbar_wait(drain, 0, p.status);
    }
  } else if (warp < 2 + kDqWarps) {
    // ---------------- dequant warps
    const int td = threadIdx.x - 64;  // 0..255
    const int col = td & 31;          // word column of the tile (gate 0..15 | up 16..31, or 0..31)
    const int jw = NPROJ == 2 ? (col >> 4) : 0;
    // rows rg, rg + 8, ... of each 64-row step; the up lanes take the
    // neighbouring row so gate and up words sit in different banks
    const int rg = (td >> 5) ^ jw;
    constexpr uint32_t M = Dq<MT>::kMagic2;
    const int64_t ngroups = K / p.group;
    const int32_t *qz = p.qz[jw];
    const uint16_t *sc = p.sc[jw];
    const int pk0 = NPROJ == 2 ? jw * (kBK * 16) + rg * 16 + (col & 15) : rg * 32 + col;
    constexpr int pk_step = NPROJ == 2 ? 8 * 16 : 8 * 32;  // words between rows r and r + 8
    // B: features col*8 .. col*8+7 -> 64-column block col/8, 16-byte chunk col%8 XOR row%8
    const int b0 = (col >> 3) * 8192 + rg * 128 + (((col & 7) ^ rg) << 4);  // + 1 KB per 8 rows
    const int spg = p.group / kBK;  // steps per group
    uint32_t act_bad = 0;  // a converted input outside F16's normal range
    // inputs in the other 16-bit dtype are converted here unless a one-time copy was made
    const bool convert = !p.preconv && p.act_dt != (std::is_same<MT, __half>::value ? MOE_F16 : MOE_BF16);
    uint32_t it = 0;
    bool live = true;
    // zeros/scales of a tile's word column
    struct ZsPtr {
      const int32_t *qz;
      const uint16_t *sc;
      bool ok;
    };
    auto zs_ptr = [&](int64_t tile) {
      const TileInfo tn = tile_info(tile);
      const int64_t wc = NPROJ == 2 ? (int64_t)tn.nt * 16 + (col & 15) : (int64_t)tn.nt * 32 + col;
      const bool ok = wc < NW;
      const int64_t wcs = ok ? wc : 0;
      return ZsPtr{qz + (int64_t)tn.e * ngroups * NW + wcs, sc + (int64_t)tn.e * ngroups * p.N + 8 * wcs, ok};
    };
    // the zero/scale rows are fetched two groups ahead, in the order the
    // loop below consumes them (the groups of a tile, then the next tile's)
    int64_t zt = blockIdx.x, zg = 0;
    ZsPtr zcur = zs_ptr(zt < total ? zt : 0);
    auto fetch = [&](uint32_t &zw, uint4 &sv) {
      zw = 0u;
      sv = make_uint4(0, 0, 0, 0);
      if (zt >= total) return;
      if (zcur.ok) {
        zw = (uint32_t)__ldg(zcur.qz + zg * NW);
        sv = __ldg(reinterpret_cast<const uint4 *>(zcur.sc + zg * p.N));
      }
      if (++zg == ngroups) {
        zg = 0;
        zt += gridDim.x;
        if (zt < total) zcur = zs_ptr(zt);
      }
    };
    uint32_t pa_zw, pb_zw;
    uint4 pa_sv, pb_sv;
    fetch(pa_zw, pa_sv);
    fetch(pb_zw, pb_sv);
    for (int64_t tile = blockIdx.x; tile < total && live; tile += gridDim.x) {
      uint32_t zp[4], sp[4];
      int gstage = 0;
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const uint32_t s = it % kLStages, ph = (it / kLStages) & 1;
        const uint32_t b = it % kBStages, buse = it / kBStages;
        if (gstage == 0) {  // a new group: take the oldest fetched zeros/scales, fetch another
          const uint32_t s4[4] = {pa_sv.x, pa_sv.y, pa_sv.z, pa_sv.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            zp[q] = nib_pair<M>(pa_zw >> (4 * q));
            sp[q] = s4[q];
          }
          pa_zw = pb_zw;
          pa_sv = pb_sv;
          fetch(pb_zw, pb_sv);
        }
        if (++gstage == spg) gstage = 0;
        if (!tc_wait(&full[s], ph, p.status, abort)) {
          live = false;
          break;
        }
        uint8_t *st = lring + s * kLBytes;
        if (convert) {
          // activation tile to the scale dtype, in place (layout-agnostic)
          uint4 *a4 = reinterpret_cast<uint4 *>(st);
#pragma unroll
          for (int i = 0; i < kABytes / 16 / 256; ++i) {
            uint4 v = a4[td + 256 * i];
            act_quad_to_mt<MT>(v, p.act_dt, act_bad);
            a4[td + 256 * i] = v;
          }
          fence_proxy_async_smem();  // the converted tile is read by the tensor core
        }
        const uint32_t *pk = reinterpret_cast<const uint32_t *>(st + kABytes) + pk0;
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = pk[i * pk_step];
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // words read (the MMA commit frees the activations)
        if (buse > 0 && !tc_wait(&bfree[b], (buse - 1) & 1, p.status, abort)) {
          live = false;
          break;
        }
        uint8_t *bt = bring + b * kBBytes + b0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint4 c;
          c.x = Dq<MT>::coef(nib_pair<M>(w[i]), zp[0], sp[0]);        // columns 0, 1
          c.y = Dq<MT>::coef(nib_pair<M>(w[i] >> 4), zp[1], sp[1]);   // columns 2, 3
          c.z = Dq<MT>::coef(nib_pair<M>(w[i] >> 8), zp[2], sp[2]);   // columns 4, 5
          c.w = Dq<MT>::coef(nib_pair<M>(w[i] >> 12), zp[3], sp[3]);  // columns 6, 7
          *reinterpret_cast<uint4 *>(bt + i * 1024) = c;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bready[b]);
      }
    }
    if (act_bad) report(p.status, MOE_DEVICE_ERR_ACT_RANGE);
  } else {
    // ---------------- epilogue warps: TMEM -> registers -> bias, rounding,
    // SwiGLU -> HBM.  The tile's bias is staged in shared memory before its
    // accumulator is waited for (one named barrier per tile, two buffers) and
    // TMEM loads are issued in pairs before one wait.  After an abort every
    // epilogue warp still runs the loop (the named barrier stays matched) but
    // reads, stores and arrives on nothing.
    const int q = warp & 3;                          // TMEM lane quarter of this warp
    const int hf = (warp - 2 - kDqWarps) >> 2;       // column half drained by this warp
    const int et = threadIdx.x - (2 + kDqWarps) * 32;  // 0 .. 255
    const bool bf = p.odt == MOE_BF16;
    uint32_t tcount = 0;
    for (int64_t tile = blockIdx.x; tile < total; tile += gridDim.x, ++tcount) {
      const TileInfo ti = tile_info(tile);
      const uint32_t buf = tcount & 1;
      float *bt = bias_s + buf * kBN;
      {  // NPROJ == 2: gate bias of the tile's 128 features, then up; else 256 columns
        const int j = NPROJ == 2 ? et >> 7 : 0;
        const int64_t n = NPROJ == 2 ? (int64_t)ti.nt * 128 + (et & 127) : (int64_t)ti.nt * kBN + et;
        bt[et] = (p.bias[j] && n < p.N) ? ld_as_float(p.bias[j], p.bias_dt, (int64_t)ti.e * p.N + n) : 0.f;
      }
      const bool ok = tc_wait(&accfull[buf], (tcount >> 1) & 1, p.status, abort);
      named_barrier(2, kEpWarps * 32);
      if (!ok) continue;
      tc_fence_after();
      const int trow = ti.mt * kBM + 32 * q + lane;  // row within the expert
      const bool row_ok = trow < ti.m && !*abort;
      const int64_t row = ti.r0 + trow;
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + buf * kBN;
      if (NPROJ == 2) {
#pragma unroll 1
        for (int c8 = 4 * hf; c8 < 4 * hf + 4; ++c8) {
          const int f0 = c8 * 16;  // feature within the tile
          uint32_t gr[16], ur[16];
          tmem_ld16_async(tbase + f0, gr);
          tmem_ld16_async(tbase + 128 + f0, ur);
          tmem_wait_ld();
          float gv[16], uv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            gv[i] = __uint_as_float(gr[i]);
            uv[i] = __uint_as_float(ur[i]);
          }
          const int64_t n0 = (int64_t)ti.nt * 128 + f0;
          if (row_ok && n0 < p.N) {
#pragma unroll
            for (int v8 = 0; v8 < 2; ++v8) {
              const float *bg = bt + f0 + 8 * v8, *bu = bt + 128 + f0 + 8 * v8;
              if (bf) finish8_bt<2, true>(p, row, n0 + 8 * v8, gv + 8 * v8, uv + 8 * v8, bg, bu);
              else finish8_bt<2, false>(p, row, n0 + 8 * v8, gv + 8 * v8, uv + 8 * v8, bg, bu);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c8 = 4 * hf; c8 < 4 * hf + 4; ++c8) {
          const int f0 = c8 * 32;
          uint32_t ra[16], rb[16];
          tmem_ld16_async(tbase + f0, ra);
          tmem_ld16_async(tbase + f0 + 16, rb);
          tmem_wait_ld();
          float yv[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            yv[i] = __uint_as_float(ra[i]);
            yv[16 + i] = __uint_as_float(rb[i]);
          }
          const int64_t n0 = (int64_t)ti.nt * 256 + f0;
          if (row_ok && n0 < p.N) {
#pragma unroll
            for (int v8 = 0; v8 < 4; ++v8) {
              const float *b8 = bt + f0 + 8 * v8;
              if (bf) finish8_bt<1, true>(p, row, n0 + 8 * v8, yv + 8 * v8, yv + 8 * v8, b8, b8);
              else finish8_bt<1, false>(p, row, n0 + 8 * v8, yv + 8 * v8, yv + 8 * v8, b8, b8);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ------------------------------------------------------------------ launch

static size_t tc_smem(int64_t E) {
  return 1024 + (size_t)tc::kLStages * tc::kLBytes + (size_t)tc::kBStages * tc::kBBytes + 256 +
         (size_t)2 * tc::kBN * 4 + (size_t)(2 * E + 1 + 32) * 4;
}

// The tile needs whole 64-row steps inside one group, 16-byte word-row
// pitches for TMA, and a 16-bit activation tile.
bool tc_fits(const ProjParams &p) {
  return p.K % tc::kBK == 0 && p.group % tc::kBK == 0 && p.N % 32 == 0 && tc_smem(p.E) <= 227 * 1024;
}

bool tc_available() { return true; }

template <typename MT, int NPROJ>
static moe_status launch_tc_t(const ProjParams &p, cudaStream_t st) {
  using namespace tc;
  CUtensorMap mx, m0, m1;
  const uint64_t NW = p.N / 8, rows = (uint64_t)p.E * p.K;
  const uint32_t box_w = NPROJ == 2 ? 16 : 32;
  // the activation map: 128-row boxes of the batch (the gather mode copies
  // its rows with cp.async and leaves the one-row map of x unused)
  const bool mx_ok = p.gather ? make_map_2d(&mx, p.x, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, p.K, p.T, kBK, 1,
                                            CU_TENSOR_MAP_SWIZZLE_128B)
                              : make_map_2d(&mx, p.x, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, p.K, p.A, kBK, kBM,
                                            CU_TENSOR_MAP_SWIZZLE_128B);
  if (!mx_ok ||
      !make_map_2d(&m0, p.qw[0], CU_TENSOR_MAP_DATA_TYPE_INT32, 4, NW, rows, box_w, kBK, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map_2d(&m1, p.qw[NPROJ - 1], CU_TENSOR_MAP_DATA_TYPE_INT32, 4, NW, rows, box_w, kBK,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return set_error(MOE_ERR_CUDA, "tensor map encoding failed (tcgen05 projection)");
  const size_t smem = tc_smem(p.E);
  auto kern = awq_fwd_tc_kernel<MT, NPROJ>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  launch_pdl(kern, dim3(num_sms()), dim3(kThreads), smem, st, mx, m0, m1, p);
  return check_launch("awq_fwd_tc_kernel");
}

moe_status launch_fwd_tc(const ProjParams &p, int nproj, bool bf16_mma, cudaStream_t st) {
  if (bf16_mma) return nproj == 2 ? launch_tc_t<__nv_bfloat16, 2>(p, st) : launch_tc_t<__nv_bfloat16, 1>(p, st);
  return nproj == 2 ? launch_tc_t<__half, 2>(p, st) : launch_tc_t<__half, 1>(p, st);
}



}  // namespace moe
