// Grouped AWQ projections on CTA pairs: one 256-row x 256-column tile per
// cluster of two SMs (tcgen05.mma.cta_group::2, M = 256), for experts whose
// batches fill 256-row tiles (long prefill batches, hot experts).
//
// ruda-tensor 0.21.34, src/packed_experts.rs -- packed_expert_forward /
//   packed_swiglu_forward (gate/up/down of the selected experts, SwiGLU);
// ruda-tensor 0.21.33, src/frozen_awq.rs -- AWQ nibble order and scale-dtype
//   coefficient rounding; the tensor-core products run in the scale dtype.
//
// Why a pair: the coefficient tile is formed in shared memory from packed
// words, so its cost (dequant instructions and shared-memory stores) is paid
// once per row tile.  With M = 256 the pair MMA reads each CTA's 128-column
// half of B for all 256 rows, so each SM dequantizes half as many
// coefficients per FLOP as a 128-row single-SM tile, and each SM's tensor
// core reads 8 KB of operands per 128 x 256 x 16 step instead of 12 KB.
//
// Split of one tile over the pair (CTA rank r = 0, 1):
//   A: rows 128 r .. 128 r + 127 of the tile, in CTA r (TMA, 128B swizzle);
//   B: output columns 128 r .. 128 r + 127 in CTA r -- for the gate/up pair
//      CTA 0 forms the gate coefficients and CTA 1 the up coefficients of the
//      same 128 features, so SwiGLU still sees G and U of a feature in one
//      TMEM lane;
//   D: rows 128 r .. of the tile, all 256 columns, in CTA r's TMEM.
// Warp roles in each CTA: warp 0 TMA producer (activations + this CTA's
// packed words, 6-stage ring); warp 1 TMEM allocation, and in CTA 0 lane 0
// issues the pair MMAs; warps 2-9 dequantize this CTA's B half (eight words
// per thread and step) into a 3-stage coefficient ring and signal CTA 0;
// warps 10-17 (two per TMEM lane quarter, one per column half) drain this
// CTA's accumulator (two TMEM buffers, so draining overlaps the next tile).
// Every wait is bounded.  CTA 1's dequant and epilogue warps arrive on CTA
// 0's barriers through the cluster shared-memory window.
#include <cudaTypedefs.h>

#include "dequant.cuh"
#include "proj.cuh"
#include "tcgen05.cuh"

namespace moe {

namespace tc2 {
constexpr int kBM = 128;   // rows per CTA (256 per pair)
constexpr int kBN = 256;   // accumulator columns
constexpr int kHalf = 128; // B columns held by each CTA
constexpr int kBK = 128;   // K per pipeline stage: two 64-element swizzle atoms
constexpr int kLStages = 3, kBStages = 3;
constexpr int kDqWarps = 8, kEpWarps = 8;
constexpr int kThreads = (2 + kDqWarps + kEpWarps) * 32;  // 576
constexpr int kRowGroups = kDqWarps * 2;                   // 16 word columns x kRowGroups threads
constexpr int kWordsPerThread = kBK / kRowGroups;          // rows rg, rg + kRowGroups, ...
constexpr int kAtom = kBM * 64 * 2;          // 16 KB: 128 rows x 64 K (128B swizzle)
constexpr int kABytes = kBM * kBK * 2;        // 32 KB
constexpr int kPBytes = kBK * (kHalf / 8) * 4;  // 8 KB packed words
constexpr int kLBytes = kABytes + kPBytes;    // one TMA stage
constexpr int kZBytes = 64;                   // zero-point words of the step's group row (16 words)
constexpr int kZSBytes = 384;                 // + its 128 scales (256 bytes), 128-byte slots
constexpr int kBBytes = kHalf * kBK * 2;      // 32 KB coefficient half-tile
constexpr int kNBlock = kBK * 128;            // bytes between 64-column blocks of B (MN-major)
constexpr int kTmemCols = 512;
}  // namespace tc2

struct PairTile {
  int e, mt, nt;
  int64_t r0;
  int m;
};

template <typename MT, int NPROJ>
__global__ void __launch_bounds__(tc2::kThreads, 1)
    awq_fwd_tc2_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w0,
                       const __grid_constant__ CUtensorMap map_w1, const __grid_constant__ CUtensorMap map_z0,
                       const __grid_constant__ CUtensorMap map_z1, const __grid_constant__ CUtensorMap map_s0,
                       const __grid_constant__ CUtensorMap map_s1, ProjParams p) {
  pdl_enter();  // programmatic dependent launch: the previous kernel is done
  using namespace tc2;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t *lring = smem;
  uint8_t *bring = smem + kLStages * kLBytes;
  uint8_t *zring = bring + kBStages * kBBytes;  // kLStages x [zero words | scales] of the step's group row
  uint64_t *lfull = reinterpret_cast<uint64_t *>(zring + kLStages * kZSBytes);
  uint64_t *lempty = lfull + kLStages;
  uint64_t *bready = lempty + kLStages;  // used in CTA 0 (both CTAs' dequant warps)
  uint64_t *bfree = bready + kBStages;
  uint64_t *accfull = bfree + kBStages;  // [2]
  uint64_t *accempty = accfull + 2;      // [2], used in CTA 0 (both CTAs' epilogues)
  uint64_t *drain = accempty + 2;        // the issuer's last commit: no MMA in flight at teardown
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int32_t *abort = reinterpret_cast<volatile int32_t *>(tmem_slot + 1);
  float *bias_s = reinterpret_cast<float *>(tmem_slot + 4);  // [2 tiles][256]: the tile's bias, staged
  int32_t *pre = reinterpret_cast<int32_t *>(bias_s + 2 * kBN);  // [E + 1]
  int32_t *cnt = pre + (p.E + 1);                             // [E]
  int32_t *tmp = cnt + p.E;                                   // [32]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int E = p.E;
  const int64_t K = p.K;
  const int feat_tile = NPROJ == 2 ? kHalf : kBN;
  const int NT = (int)((p.N + feat_tile - 1) / feat_tile);
  const int nk = (int)(K / kBK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLStages; ++s) {
      mbar_init(&lfull[s], p.gather ? 1 + 32 : 1);  // + the producer lanes' gathered rows
      mbar_init(&lempty[s], 1 + kDqWarps);  // pair-MMA commit + this CTA's dequant warps
    }
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&bready[s], 2 * kDqWarps);
      mbar_init(&bfree[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], 2 * kEpWarps);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int32_t a = p.offsets[e], b = p.offsets[e + 1];
    const bool bad = a < 0 || b < a || (int64_t)b > p.A || (e == 0 && a != 0) || (e == E - 1 && (int64_t)b != p.A);
    if (bad && blockIdx.x == 0) report(p.status, MOE_DEVICE_ERR_OFFSETS);
    cnt[e] = bad ? 0 : NT * ((b - a + 2 * kBM - 1) / (2 * kBM));
  }
  __syncthreads();
  block_exclusive_scan(cnt, E, pre, tmp);
  const int64_t total = pre[E];
  if (pair >= total) return;  // same answer in both CTAs of the pair

  auto tile_info = [&](int64_t tile) {
    PairTile ti;
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

  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer: this CTA's activation rows and packed half
    // (lane 0, by TMA).  With a gather, every lane copies four rows of each
    // activation step with 16-byte cp.async into the swizzled atoms (lane L:
    // tile rows L, L + 32, L + 64, L + 96), and arrives on the stage's full
    // barrier once its copies of that stage landed (one stage behind, so two
    // stages stay in flight), after a proxy fence for the tensor core.
    const bool gather = p.gather != nullptr;
    if (gather || lane == 0) {
      const CUtensorMap *mw = (NPROJ == 2 && rank == 1) ? &map_w1 : &map_w0;
      const CUtensorMap *mz = (NPROJ == 2 && rank == 1) ? &map_z1 : &map_z0;
      const CUtensorMap *ms = (NPROJ == 2 && rank == 1) ? &map_s1 : &map_s0;
      const int64_t ngroups = K / p.group;
      // shared-memory offsets of this lane's 16-byte chunks inside an atom
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
        mbar_arrive(&lfull[pend_s]);
        pend = false;
      };
      for (int64_t tile = pair; tile < total && live; tile += npairs) {
        const PairTile ti = tile_info(tile);
        const int32_t row0 = (int32_t)(ti.r0 + (int64_t)ti.mt * 2 * kBM + kBM * rank);
        const int32_t wcol = NPROJ == 2 ? ti.nt * 16 : ti.nt * 32 + 16 * (int)rank;
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
            ok = use == 0 || tc_wait(&lempty[s], (use - 1) & 1, p.status, abort);
            if (ok) mbar_arrive_expect_tx(&lfull[s], (gather ? kPBytes : kLBytes) + kZBytes + 256);
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
              for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int cc = 0; cc < 8; ++cc)
                  cp_async16(sbase + a * kAtom + i * 4096 + ((cc ^ (lane & 7)) << 4), src + a * 64 + cc * 8);
            }
            cp_async_commit();
            deliver(false);  // the previous stage (at most this one's copies left in flight)
            pend = true;
            pend_s = s;
          }
          if (lane == 0) {
            if (!gather) {
              tma_load_2d(st, &map_x, &lfull[s], kb * kBK, row0);
              tma_load_2d(st + kAtom, &map_x, &lfull[s], kb * kBK + 64, row0);
            }
            tma_load_2d(st + kABytes, mw, &lfull[s], wcol, (int32_t)(ti.e * K + (int64_t)kb * kBK));
            // the group row of this step's zero points and scales (this CTA's columns)
            const int32_t grow = (int32_t)(ti.e * ngroups + (int64_t)kb * kBK / p.group);
            uint8_t *zs = zring + s * kZSBytes;
            tma_load_2d(zs, mz, &lfull[s], wcol, grow);
            tma_load_2d(zs + 128, ms, &lfull[s], wcol * 8, grow);
          }
        }
      }
      if (gather) deliver(true);  // every issued stage complete before the drain below
      if (lane == 0) tma_drain(lfull, it, kLStages, p.status);
    }
  } else if (warp == 1) {
    // ---------------- pair MMA issuer (CTA 0 only)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t fmt = std::is_same<MT, __half>::value ? 0u : 1u;
      // D F32, A/B in the scale dtype, A K-major, B MN-major, N = 256, M = 256
      const uint32_t idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | (1u << 16) | ((uint32_t)(kBN >> 3) << 17) |
                             ((uint32_t)((2 * kBM) >> 4) << 24);
      uint32_t it = 0, tcount = 0;
      bool live = true;
      for (int64_t tile = pair; tile < total; tile += npairs, ++tcount) {
        const uint32_t buf = tcount & 1, use = tcount >> 1;
        if (use > 0 && !tc_wait_cluster(&accempty[buf], (use - 1) & 1, p.status, abort)) break;
        tc_fence_after();
        const uint32_t dacc = tmem + buf * kBN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t ls = it % kLStages, bs = it % kBStages;
          // both CTAs' dequant warps arrive only after their own TMA stage landed
          if (!tc_wait_cluster(&bready[bs], (it / kBStages) & 1, p.status, abort)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(lring + ls * kLBytes);
          const uint64_t bdesc = smem_desc(smem_u32(bring + bs * kBBytes), kNBlock, 1024);
#pragma unroll
          for (int j = 0; j < kBK / 16; ++j)  // K steps of 16: atom j / 4, 32 bytes each inside it
            umma2_f16(dacc, smem_desc(a_addr + (j >> 2) * kAtom, 16, 1024) + (uint64_t)(2 * (j & 3)),
                      bdesc + (uint64_t)(128 * j), idesc, (kb | j) != 0);
          umma2_commit_both(&lempty[ls]);
          umma2_commit_both(&bfree[bs]);
        }
        if (!live) break;
        umma2_commit_both(&accfull[buf]);
      }
      umma2_commit_both(drain);  // arrives in both CTAs once every MMA issued above has completed
    }
    if (lane == 0) mbar_wait(drain, 0, p.status);
  } else if (warp < 2 + kDqWarps) {
    // ---------------- dequant warps: this CTA's 128-column half of B
    const int td = threadIdx.x - 64;  // 0 .. 32 kDqWarps - 1
    const int col = td & 15;          // word column within the half
    const int rg = td >> 4;           // rows rg, rg + kRowGroups, ... of each step
    constexpr uint32_t M = Dq<MT>::kMagic2;
    const int pk0 = rg * 16 + col;
    // features col*8 .. col*8+7 of the half -> 64-column block col/8, 16-byte
    // chunk col%8 XOR row%8 (MN-major, 128-byte swizzle, 8-row x 64-column atoms)
    const int b0 = (col >> 3) * kNBlock + (rg >> 3) * 1024 + (rg & 7) * 128 + (((col & 7) ^ (rg & 7)) << 4);
    const int spg = p.group / kBK;
    uint32_t act_bad = 0;  // a converted input outside F16's normal range
    // inputs in the other 16-bit dtype are converted here unless a one-time copy was made
    const bool convert = !p.preconv && p.act_dt != (std::is_same<MT, __half>::value ? MOE_F16 : MOE_BF16);
    uint64_t *bready0 = bready;  // CTA 0's barriers, addressed through the cluster window
    uint32_t it = 0;
    bool live = true;
    for (int64_t tile = pair; tile < total && live; tile += npairs) {
      uint32_t zp[4], sp[4];
      int gstage = 0;
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const uint32_t ls = it % kLStages, bs = it % kBStages, buse = it / kBStages;
        if (!tc_wait(&lfull[ls], (it / kLStages) & 1, p.status, abort)) {
          live = false;
          break;
        }
        uint8_t *st = lring + ls * kLBytes;
        if (gstage == 0) {  // a new group: its zero/scale row came with this stage
          const uint8_t *zs = zring + ls * kZSBytes;
          const uint32_t zw = reinterpret_cast<const uint32_t *>(zs)[col];
          const uint4 sv = reinterpret_cast<const uint4 *>(zs + 128)[col];
          const uint32_t s4[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            zp[q] = nib_pair<M>(zw >> (4 * q));
            sp[q] = s4[q];
          }
        }
        if (++gstage == spg) gstage = 0;
        uint32_t w[kWordsPerThread];
        {
          const uint32_t *pk = reinterpret_cast<const uint32_t *>(st + kABytes) + pk0;
#pragma unroll
          for (int i = 0; i < kWordsPerThread; ++i) w[i] = pk[i * kRowGroups * 16];
        }
        if (convert) {
          uint4 *a4 = reinterpret_cast<uint4 *>(st);
#pragma unroll
          for (int i = 0; i < kABytes / 16 / (32 * kDqWarps); ++i) {
            uint4 v = a4[td + 32 * kDqWarps * i];
            act_quad_to_mt<MT>(v, p.act_dt, act_bad);
            a4[td + 32 * kDqWarps * i] = v;
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&lempty[ls]);  // packed words read (the pair commit frees A)
        if (buse > 0 && !tc_wait(&bfree[bs], (buse - 1) & 1, p.status, abort)) {
          live = false;
          break;
        }
        uint8_t *bt = bring + bs * kBBytes + b0;
#pragma unroll
        for (int i = 0; i < kWordsPerThread; ++i) {
          uint4 c;
          c.x = Dq<MT>::coef(nib_pair<M>(w[i]), zp[0], sp[0]);
          c.y = Dq<MT>::coef(nib_pair<M>(w[i] >> 4), zp[1], sp[1]);
          c.z = Dq<MT>::coef(nib_pair<M>(w[i] >> 8), zp[2], sp[2]);
          c.w = Dq<MT>::coef(nib_pair<M>(w[i] >> 12), zp[3], sp[3]);
          *reinterpret_cast<uint4 *>(bt + i * kRowGroups * 128) = c;  // rows + kRowGroups
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(cluster_addr(&bready0[bs], 0));
      }
    }
    if (act_bad) report(p.status, MOE_DEVICE_ERR_ACT_RANGE);
  } else {
    // ---------------- epilogue warps: this CTA's 128 rows of the tile.  The
    // tile's bias is staged in shared memory before its accumulator is
    // waited for (one named barrier per tile, two buffers), and TMEM loads
    // are issued in pairs before one wait.  After an abort every epilogue
    // warp still runs the loop (the named barrier stays matched) but reads,
    // stores and arrives on nothing.
    const int q = warp & 3;                     // TMEM lane quarter
    const int hf = (warp - 2 - kDqWarps) >> 2;  // column half drained by this warp
    const int et = threadIdx.x - (2 + kDqWarps) * 32;  // 0 .. 255
    const bool bf = p.odt == MOE_BF16;
    uint32_t tcount = 0;
    for (int64_t tile = pair; tile < total; tile += npairs, ++tcount) {
      const PairTile ti = tile_info(tile);
      const uint32_t buf = tcount & 1;
      float *bt = bias_s + buf * kBN;
      {  // NPROJ == 2: gate bias of the tile's 128 features, then up; else 256 columns
        const int j = NPROJ == 2 ? et >> 7 : 0;
        const int64_t n = NPROJ == 2 ? (int64_t)ti.nt * kHalf + (et & (kHalf - 1)) : (int64_t)ti.nt * kBN + et;
        bt[et] = (p.bias[j] && n < p.N) ? ld_as_float(p.bias[j], p.bias_dt, (int64_t)ti.e * p.N + n) : 0.f;
      }
      const bool ok = tc_wait(&accfull[buf], (tcount >> 1) & 1, p.status, abort);
      named_barrier(2, kEpWarps * 32);
      if (!ok) continue;
      tc_fence_after();
      const int trow = ti.mt * 2 * kBM + kBM * (int)rank + 32 * q + lane;
      const bool row_ok = trow < ti.m && !*abort;
      const int64_t row = ti.r0 + trow;
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + buf * kBN;
      if (NPROJ == 2) {
#pragma unroll 1
        for (int c8 = 4 * hf; c8 < 4 * hf + 4; ++c8) {
          const int f0 = c8 * 16;
          uint32_t gr[16], ur[16];
          tmem_ld16_async(tbase + f0, gr);
          tmem_ld16_async(tbase + kHalf + f0, ur);
          tmem_wait_ld();
          float gv[16], uv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            gv[i] = __uint_as_float(gr[i]);
            uv[i] = __uint_as_float(ur[i]);
          }
          const int64_t n0 = (int64_t)ti.nt * kHalf + f0;
          if (row_ok && n0 < p.N) {
#pragma unroll
            for (int v8 = 0; v8 < 2; ++v8) {
              const float *bg = bt + f0 + 8 * v8, *bu = bt + kHalf + f0 + 8 * v8;
              if (bf) finish8_bt<2, true>(p, row, n0 + 8 * v8, gv + 8 * v8, uv + 8 * v8, bg, bu);
              else finish8_bt<2, false>(p, row, n0 + 8 * v8, gv + 8 * v8, uv + 8 * v8, bg, bu);
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c32 = 4 * hf; c32 < 4 * hf + 4; ++c32) {
          const int f0 = c32 * 32;
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
          const int64_t n0 = (int64_t)ti.nt * kBN + f0;
          if (row_ok && n0 < p.N) {
#pragma unroll
            for (int v8 = 0; v8 < 4; ++v8) {
              if (n0 + 8 * v8 >= p.N) break;
              const float *b8 = bt + f0 + 8 * v8;
              if (bf) finish8_bt<1, true>(p, row, n0 + 8 * v8, yv + 8 * v8, yv + 8 * v8, b8, b8);
              else finish8_bt<1, false>(p, row, n0 + 8 * v8, yv + 8 * v8, yv + 8 * v8, b8, b8);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_addr(&accempty[buf], 0));
    }
  }
  // Neither CTA leaves while its peer may still read its shared memory or
  // arrive on its barriers; then both release the pair's TMEM.
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ------------------------------------------------------------------ launch

static size_t tc2_smem(int64_t E) {
  return 1024 + (size_t)tc2::kLStages * tc2::kLBytes + (size_t)tc2::kBStages * tc2::kBBytes +
         (size_t)tc2::kLStages * tc2::kZSBytes + 256 + (size_t)2 * tc2::kBN * 4 + (size_t)(2 * E + 1 + 32) * 4;
}

bool tc2_fits(const ProjParams &p) {
  return p.K % tc2::kBK == 0 && p.group % tc2::kBK == 0 && p.N % 32 == 0 && tc2_smem(p.E) <= 227 * 1024;
}

template <typename MT, int NPROJ>
static moe_status launch_tc2_t(const ProjParams &p, cudaStream_t st) {
  using namespace tc2;
  CUtensorMap mx, m0, m1;
  const uint64_t NW = p.N / 8, rows = (uint64_t)p.E * p.K;
  // the activation map: 128-row boxes of the batch (the gather mode copies
  // its rows with cp.async and leaves the one-row map of x unused)
  const bool mx_ok = p.gather ? make_map_2d(&mx, p.x, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, p.K, p.T, 64, 1,
                                            CU_TENSOR_MAP_SWIZZLE_128B)
                              : make_map_2d(&mx, p.x, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, p.K, p.A, 64, kBM,
                                            CU_TENSOR_MAP_SWIZZLE_128B);
  // zero-point words and scales: one group row per step, this CTA's 16 word columns
  CUtensorMap z0, z1, s0, s1;
  const uint64_t grows = (uint64_t)p.E * (p.K / p.group);
  if (!mx_ok ||
      !make_map_2d(&m0, p.qw[0], CU_TENSOR_MAP_DATA_TYPE_INT32, 4, NW, rows, 16, kBK, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map_2d(&m1, p.qw[NPROJ - 1], CU_TENSOR_MAP_DATA_TYPE_INT32, 4, NW, rows, 16, kBK,
                   CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map_2d(&z0, p.qz[0], CU_TENSOR_MAP_DATA_TYPE_INT32, 4, NW, grows, 16, 1, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map_2d(&z1, p.qz[NPROJ - 1], CU_TENSOR_MAP_DATA_TYPE_INT32, 4, NW, grows, 16, 1,
                   CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map_2d(&s0, p.sc[0], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, p.N, grows, 128, 1, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map_2d(&s1, p.sc[NPROJ - 1], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, p.N, grows, 128, 1,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return set_error(MOE_ERR_CUDA, "tensor map encoding failed (tcgen05 pair projection)");
  const size_t smem = tc2_smem(p.E);
  auto kern = awq_fwd_tc2_kernel<MT, NPROJ>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_pdl
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(2 * (num_sms() / 2));
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) {
    cudaGetLastError();
    return set_error(MOE_ERR_CUDA, "no co-resident SM pair for the tcgen05 pair projection");
  }
  cfg.gridDim = dim3(2 * clusters);  // persistent: every pair resident at once
  cfg.numAttrs = 2;
  cudaLaunchKernelEx(&cfg, kern, mx, m0, m1, z0, z1, s0, s1, p);
  return check_launch("awq_fwd_tc2_kernel");
}

moe_status launch_fwd_tc2(const ProjParams &p, int nproj, bool bf16_mma, cudaStream_t st) {
  if (bf16_mma) return nproj == 2 ? launch_tc2_t<__nv_bfloat16, 2>(p, st) : launch_tc2_t<__nv_bfloat16, 1>(p, st);
  return nproj == 2 ? launch_tc2_t<__half, 2>(p, st) : launch_tc2_t<__half, 1>(p, st);
}

}  // namespace moe
