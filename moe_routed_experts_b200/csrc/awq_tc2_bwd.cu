// Frozen input VJP on CTA pairs: dinput = RNE(grad . W^T (+ grad2 . W2^T))
// for experts whose batches fill 256-row tiles (long prefill batches, hot
// experts).
//
// ruda-tensor 0.21.34, src/packed_experts.rs -- packed_expert_input_backward /
//   packed_swiglu_input_backward (the gate and up contributions summed
//   before one rounding);
// ruda-tensor 0.21.33, src/frozen_awq.rs -- FrozenAwqOps input backward: the
//   transpose of the same scale-dtype coefficients, no weight gradients.
//
// Tile per cluster of two SMs: 256 gradient rows x 256 output columns kk,
// reduction over the forward output width n in steps of 128.  CTA r holds
// gradient rows 128 r .. 128 r + 127 (TMA, two 128B-swizzled atoms per
// step), and forms the coefficients of output columns kk0 + 128 r .. + 127:
// a packed word of row kk holds 8 consecutive n, so each dequantized word is
// one 16-byte chunk of a K-major (reduction-contiguous) B row.  The pair MMA
// (tcgen05.mma.cta_group::2, M = 256, N = 256) leaves row 128 r + i, all 256
// output columns, in lane i of CTA r's TMEM.  Warp roles and barriers follow
// the forward pair tile: warp 0 TMA producer (gradient, packed words, and
// the zero/scale rows of the step), warp 1 TMEM + (CTA 0) MMA issue, warps
// 2-17 dequantize, warps 18-25 (two per TMEM lane quarter) drain the
// double-buffered accumulator.
#include <cudaTypedefs.h>

#include "dequant.cuh"
#include "proj.cuh"
#include "tcgen05.cuh"

namespace moe {

namespace tc2b {
constexpr int kBM = 128;   // gradient rows per CTA
constexpr int kBN = 256;   // output columns per pair tile
constexpr int kHalf = 128; // output columns formed by each CTA
constexpr int kBK = 128;   // reduction per stage (16 words)
constexpr int kLStages = 3, kBStages = 3;
constexpr int kDqWarps = 16, kEpWarps = 8;
constexpr int kThreads = (2 + kDqWarps + kEpWarps) * 32;  // 832
constexpr int kAtom = kBM * 64 * 2;                       // 16 KB: 128 rows x 64 (128B swizzle)
constexpr int kABytes = kBM * kBK * 2;                    // 32 KB gradient tile
constexpr int kPBytes = kHalf * (kBK / 8) * 4;            // 8 KB packed words (128 rows x 16 words)
constexpr int kZBytes = 2 * (kBK / 8) * 4;                // zero words: up to 2 group rows x 16 words
constexpr int kCBytes = 1024;                             // zero + scale rows (padded)
constexpr int kLBytes = kABytes + kPBytes + kCBytes;      // 41 KB
constexpr int kBAtom = kHalf * 64 * 2;                    // 16 KB: 128 rows x 64 reduction indices
constexpr int kBBytes = kHalf * kBK * 2;                  // 32 KB
constexpr int kTmemCols = 512;
}  // namespace tc2b

struct PairBwdTile {
  int e, mt, ct;
  int64_t r0;
  int m;
};

struct PairBwdMaps {
  CUtensorMap grad[2], qw[2], qz[2], sc[2];
};

template <typename MT, int NPROJ>
__global__ void __launch_bounds__(tc2b::kThreads, 1)
    awq_bwd_tc2_kernel(const __grid_constant__ PairBwdMaps maps, BwdParams p) {
  using namespace tc2b;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t *lring = smem;
  uint8_t *bring = smem + kLStages * kLBytes;
  uint64_t *lfull = reinterpret_cast<uint64_t *>(bring + kBStages * kBBytes);
  uint64_t *lempty = lfull + kLStages;
  uint64_t *bready = lempty + kLStages;  // used in CTA 0
  uint64_t *bfree = bready + kBStages;
  uint64_t *accfull = bfree + kBStages;  // [2]
  uint64_t *accempty = accfull + 2;      // [2], used in CTA 0
  uint64_t *drain = accempty + 2;        // the issuer's last commit: no MMA in flight at teardown
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int32_t *abort = reinterpret_cast<volatile int32_t *>(tmem_slot + 1);
  int32_t *pre = reinterpret_cast<int32_t *>(tmem_slot + 4);  // [E + 1]
  int32_t *cnt = pre + (p.E + 1);                             // [E]
  int32_t *tmp = cnt + p.E;                                   // [32]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int E = p.E;
  const int64_t K = p.K, N = p.N;
  const int CT = (int)((K + kBN - 1) / kBN);
  const int nkp = (int)(N / kBK);
  const int nk = NPROJ * nkp;
  const int grows = p.group >= kHalf ? 1 : kHalf / p.group;  // group rows of a CTA's 128 output columns
  const uint32_t stage_tx = kABytes + kPBytes + grows * ((kBK / 8) * 4 + kBK * 2);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLStages; ++s) {
      mbar_init(&lfull[s], 1);
      mbar_init(&lempty[s], 1 + kDqWarps);
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
    cnt[e] = bad ? 0 : CT * ((b - a + 2 * kBM - 1) / (2 * kBM));
  }
  __syncthreads();
  block_exclusive_scan(cnt, E, pre, tmp);
  const int64_t total = pre[E];
  if (pair >= total) return;  // same answer in both CTAs of the pair

  auto tile_info = [&](int64_t tile) {
    PairBwdTile ti;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= tile) lo = mid;
      else hi = mid - 1;
    }
    ti.e = lo;
    const int64_t local = tile - pre[lo];
    ti.mt = (int)(local / CT);
    ti.ct = (int)(local % CT);
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
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer: gradient rows, packed half, zero/scale rows
    if (lane == 0) {
      uint32_t it = 0;  // stages issued
      bool live = true;
      for (int64_t tile = pair; tile < total && live; tile += npairs) {
        const PairBwdTile ti = tile_info(tile);
        const int32_t row0 = (int32_t)(ti.r0 + (int64_t)ti.mt * 2 * kBM + kBM * rank);
        const int64_t kk0 = (int64_t)ti.ct * kBN + kHalf * rank;  // this CTA's first output column
        const int32_t wrow = (int32_t)(ti.e * K + kk0);
        const int32_t grow = (int32_t)((ti.e * K + kk0) / p.group);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t s = it % kLStages, use = it / kLStages;
          if (use > 0 && !tc_wait(&lempty[s], (use - 1) & 1, p.status, abort)) {
            live = false;
            break;
          }
          const int j = NPROJ == 2 ? kb / nkp : 0;
          const int32_t n0 = (kb - j * nkp) * kBK;
          uint8_t *st = lring + s * kLBytes;
          uint8_t *cs = st + kABytes + kPBytes;
          mbar_arrive_expect_tx(&lfull[s], stage_tx);
          tma_load_2d(st, &maps.grad[j], &lfull[s], n0, row0);
          tma_load_2d(st + kAtom, &maps.grad[j], &lfull[s], n0 + 64, row0);
          tma_load_2d(st + kABytes, &maps.qw[j], &lfull[s], n0 / 8, wrow);
          tma_load_2d(cs, &maps.qz[j], &lfull[s], n0 / 8, grow);
          tma_load_2d(cs + kZBytes, &maps.sc[j], &lfull[s], n0, grow);
        }
      }
      tma_drain(lfull, it, kLStages, p.status);
    }
  } else if (warp == 1) {
    // ---------------- pair MMA issuer (CTA 0 only)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t fmt = std::is_same<MT, __half>::value ? 0u : 1u;
      // D F32, A/B in the scale dtype, both K-major, N = 256, M = 256
      const uint32_t idesc =
          (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)((2 * kBM) >> 4) << 24);
      uint32_t it = 0, tcount = 0;
      bool live = true;
      for (int64_t tile = pair; tile < total; tile += npairs, ++tcount) {
        const uint32_t buf = tcount & 1, use = tcount >> 1;
        if (use > 0 && !tc_wait_cluster(&accempty[buf], (use - 1) & 1, p.status, abort)) break;
        tc_fence_after();
        const uint32_t dacc = tmem + buf * kBN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t ls = it % kLStages, bs = it % kBStages;
          if (!tc_wait_cluster(&bready[bs], (it / kBStages) & 1, p.status, abort)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(lring + ls * kLBytes);
          const uint32_t b_addr = smem_u32(bring + bs * kBBytes);
#pragma unroll
          for (int jj = 0; jj < kBK / 16; ++jj)  // 16-deep steps: atom jj / 4, 32 bytes each inside it
            umma2_f16(dacc, smem_desc(a_addr + (jj >> 2) * kAtom, 16, 1024) + (uint64_t)(2 * (jj & 3)),
                      smem_desc(b_addr + (jj >> 2) * kBAtom, 16, 1024) + (uint64_t)(2 * (jj & 3)), idesc,
                      (kb | jj) != 0);
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
    // ---------------- dequant warps: 128 output columns x 16 words per step
    const int td = threadIdx.x - 64;  // 0..511
    const int wcol = td & 15;         // word: reduction indices 8 wcol .. 8 wcol + 7 of the step
    const int rband = td >> 4;        // output rows rband + 32 i, i = 0..3
    constexpr uint32_t M = Dq<MT>::kMagic2;
    // K-major B: row r at atom (wcol / 8), chunk (wcol % 8) XOR (r % 8)
    const int b0 = (wcol >> 3) * kBAtom + (rband >> 3) * 1024 + (rband & 7) * 128 + (((wcol & 7) ^ (rband & 7)) << 4);
    const int gshift = p.group >= kHalf ? 8 : 6;  // group row of band i: (32 i) >> gshift (groups 64 or >= 128)
    uint32_t act_bad = 0;  // a converted input outside F16's normal range
    // gradients in the other 16-bit dtype are converted here unless a one-time copy was made
    const bool convert = !p.preconv && p.gdt != (std::is_same<MT, __half>::value ? MOE_F16 : MOE_BF16);
    uint64_t *bready0 = bready;
    uint32_t it = 0;
    bool live = true;
    for (int64_t tile = pair; tile < total && live; tile += npairs) {
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const uint32_t ls = it % kLStages, bs = it % kBStages, buse = it / kBStages;
        if (!tc_wait(&lfull[ls], (it / kLStages) & 1, p.status, abort)) {
          live = false;
          break;
        }
        uint8_t *st = lring + ls * kLBytes;
        const uint32_t *pk = reinterpret_cast<const uint32_t *>(st + kABytes) + rband * 16 + wcol;
        const uint8_t *cs = st + kABytes + kPBytes;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = pk[i * 32 * 16];
        // the (at most two) group rows of this CTA's columns
        const uint32_t zw0 = reinterpret_cast<const uint32_t *>(cs)[wcol];
        const uint32_t zw1 = reinterpret_cast<const uint32_t *>(cs)[16 + wcol];
        const uint4 sv0 = *reinterpret_cast<const uint4 *>(cs + kZBytes + wcol * 16);
        const uint4 sv1 = *reinterpret_cast<const uint4 *>(cs + kZBytes + kBK * 2 + wcol * 16);
        if (convert) {
          uint4 *a4 = reinterpret_cast<uint4 *>(st);
#pragma unroll
          for (int i = 0; i < kABytes / 16 / (32 * kDqWarps); ++i) {
            uint4 v = a4[td + 32 * kDqWarps * i];
            act_quad_to_mt<MT>(v, p.gdt, act_bad);
            a4[td + 32 * kDqWarps * i] = v;
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&lempty[ls]);  // packed words and constants read
        if (buse > 0 && !tc_wait(&bfree[bs], (buse - 1) & 1, p.status, abort)) {
          live = false;
          break;
        }
        uint8_t *bt = bring + bs * kBBytes + b0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const bool g1 = ((32 * i) >> gshift) != 0;  // second group row (groups of 64)
          const uint32_t zw = g1 ? zw1 : zw0;
          const uint4 sv = g1 ? sv1 : sv0;
          uint4 c;
          c.x = Dq<MT>::coef(nib_pair<M>(w[i]), nib_pair<M>(zw), sv.x);               // n 0, 1
          c.y = Dq<MT>::coef(nib_pair<M>(w[i] >> 4), nib_pair<M>(zw >> 4), sv.y);     // n 2, 3
          c.z = Dq<MT>::coef(nib_pair<M>(w[i] >> 8), nib_pair<M>(zw >> 8), sv.z);     // n 4, 5
          c.w = Dq<MT>::coef(nib_pair<M>(w[i] >> 12), nib_pair<M>(zw >> 12), sv.w);   // n 6, 7
          *reinterpret_cast<uint4 *>(bt + i * 4096) = c;                                   // rows + 32
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(cluster_addr(&bready0[bs], 0));
      }
    }
    if (act_bad) report(p.status, MOE_DEVICE_ERR_ACT_RANGE);
  } else {
    // ---------------- epilogue warps: this CTA's 128 rows, 256 output columns
    const int q = warp & 3;                     // TMEM lane quarter
    const int hf = (warp - 2 - kDqWarps) >> 2;  // column half drained by this warp
    const bool bf = p.odt == MOE_BF16;
    uint32_t tcount = 0;
    for (int64_t tile = pair; tile < total; tile += npairs, ++tcount) {
      const PairBwdTile ti = tile_info(tile);
      const uint32_t buf = tcount & 1;
      if (!tc_wait(&accfull[buf], (tcount >> 1) & 1, p.status, abort)) break;
      tc_fence_after();
      const int trow = ti.mt * 2 * kBM + kBM * (int)rank + 32 * q + lane;
      const bool row_ok = trow < ti.m && !*abort;
      const int64_t row = ti.r0 + trow;
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + buf * kBN;
#pragma unroll 1
      for (int c16 = 8 * hf; c16 < 8 * hf + 8; ++c16) {
        float v[16];
        tmem_ld16(tbase + c16 * 16, v);
        const int64_t kk = (int64_t)ti.ct * kBN + c16 * 16;
        if (row_ok && kk < K) {
          uint32_t o[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            o[i] = bf ? round_pair<true>(v[2 * i], v[2 * i + 1]) : round_pair<false>(v[2 * i], v[2 * i + 1]);
          uint4 *dst = reinterpret_cast<uint4 *>(p.out + row * K + kk);
          dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
          dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_addr(&accempty[buf], 0));
    }
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ------------------------------------------------------------------ launch

static size_t tc2b_smem(int64_t E) {
  return 1024 + (size_t)tc2b::kLStages * tc2b::kLBytes + (size_t)tc2b::kBStages * tc2b::kBBytes + 256 +
         (size_t)(2 * E + 1 + 32) * 4;
}

// Whole 128-wide reduction steps, 16-column output chunks, and groups of 64
// or a multiple of 128 (at most two group rows per CTA's 128 columns).
bool tc2_bwd_fits(const BwdParams &p) {
  const bool groups_ok = p.group == 64 || p.group % 128 == 0;
  return p.N % tc2b::kBK == 0 && p.K % 16 == 0 && groups_ok && tc2b_smem(p.E) <= 227 * 1024;
}

template <typename MT, int NPROJ>
static moe_status launch_bwd_tc2_t(const BwdParams &p, cudaStream_t st) {
  using namespace tc2b;
  PairBwdMaps maps;
  const uint64_t NW = p.N / 8, rows = (uint64_t)p.E * p.K, grows_all = rows / p.group;
  const uint32_t gbox = p.group >= kHalf ? 1 : kHalf / p.group;
  for (int j = 0; j < 2; ++j) {
    const int jj = j < NPROJ ? j : 0;
    if (!make_map_2d(&maps.grad[j], p.grad[jj], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, p.N, p.A, 64, kBM,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&maps.qw[j], p.qw[jj], CU_TENSOR_MAP_DATA_TYPE_INT32, 4, NW, rows, kBK / 8, kHalf,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map_2d(&maps.qz[j], p.qz[jj], CU_TENSOR_MAP_DATA_TYPE_INT32, 4, NW, grows_all, kBK / 8, gbox,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map_2d(&maps.sc[j], p.sc[jj], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, p.N, grows_all, kBK, gbox,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
      return set_error(MOE_ERR_CUDA, "tensor map encoding failed (tcgen05 pair input VJP)");
  }
  const size_t smem = tc2b_smem(p.E);
  auto kern = awq_bwd_tc2_kernel<MT, NPROJ>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(2 * (num_sms() / 2));
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1) {
    cudaGetLastError();
    return set_error(MOE_ERR_CUDA, "no co-resident SM pair for the tcgen05 pair input VJP");
  }
  cfg.gridDim = dim3(2 * clusters);
  cudaLaunchKernelEx(&cfg, kern, maps, p);
  return check_launch("awq_bwd_tc2_kernel");
}

moe_status launch_bwd_tc2(const BwdParams &p, int nproj, bool bf16_mma, cudaStream_t st) {
  if (bf16_mma)
    return nproj == 2 ? launch_bwd_tc2_t<__nv_bfloat16, 2>(p, st) : launch_bwd_tc2_t<__nv_bfloat16, 1>(p, st);
  return nproj == 2 ? launch_bwd_tc2_t<__half, 2>(p, st) : launch_bwd_tc2_t<__half, 1>(p, st);
}

}  // namespace moe
