// Frozen input VJP of the grouped AWQ projections on tcgen05 tensor cores:
// dinput[r, kk] = RNE( sum_n grad[r, n] W[e, kk, n] (+ sum_n grad2[r, n] W2[e, kk, n]) )
// with the same scale-dtype coefficients W as the forward, transposed.
//
// ruda-tensor 0.21.34, src/packed_experts.rs -- packed_expert_input_backward /
//   packed_swiglu_input_backward (input VJP of the frozen expert bank; the
//   gate and up contributions summed before one rounding);
// ruda-tensor 0.21.33, src/frozen_awq.rs -- FrozenAwqOps input backward: the
//   transpose of the same rounded coefficients, no weight gradients.
//
// As a GEMM per expert: D[rows x K] = G[rows x N] . W^T, reduction over the
// forward output width N.  A packed word holds 8 consecutive reduction
// indices n of one output column kk, so the coefficient tile is built
// K-major (reduction-contiguous): the dequantized word is one 16-byte chunk
// of a B row.  Tile: 128 rows x 256 output columns, reduction in steps of 64
// (8 word columns); the gate/up pair simply continues the reduction over the
// second (grad, payload).  Warp roles as in the forward tile: warp 0 TMA
// producer (gradient tile, packed words, and the zero/scale rows of the
// step, 3-stage ring); warp 1 TMEM allocation + single-thread MMA issue;
// warps 2-9 dequantize; warps 10-17 (two per TMEM lane quarter) drain a
// double-buffered TMEM accumulator, round once to the gradient dtype and
// store.
#include <cudaTypedefs.h>

#include "dequant.cuh"
#include "proj.cuh"
#include "tcgen05.cuh"

namespace moe {

namespace tcb {
constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 3;
constexpr int kDqWarps = 8, kEpWarps = 8;
constexpr int kThreads = (2 + kDqWarps + kEpWarps) * 32;  // 576
constexpr int kABytes = kBM * kBK * 2;     // 16 KB gradient tile
constexpr int kBBytes = kBN * kBK * 2;     // 32 KB coefficient tile (256 rows x 128 B)
constexpr int kPBytes = kBN * (kBK / 8) * 4;  // 8 KB packed words (256 rows x 8 words)
constexpr int kZBytes = 4 * 8 * 4;         // zero words: up to 4 group rows x 8 words
constexpr int kCBytes = 1024;              // zero + scale region (padded)
constexpr int kStageBytes = kABytes + kBBytes + kPBytes + kCBytes;
constexpr int kTmemCols = 512;
}  // namespace tcb

struct BwdMaps {
  CUtensorMap grad[2], qw[2], qz[2], sc[2];
};

struct BwdTile {
  int e, mt, ct;
  int64_t r0;
  int m;
};

template <typename MT, int NPROJ>
__global__ void __launch_bounds__(tcb::kThreads, 1)
    awq_bwd_tc_kernel(const __grid_constant__ BwdMaps maps, BwdParams p) {
  using namespace tcb;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t *stages = smem;  // kStages x [A | B | packed | zeros, scales]
  uint64_t *full = reinterpret_cast<uint64_t *>(stages + kStages * kStageBytes);
  uint64_t *bready = full + kStages;
  uint64_t *empty = bready + kStages;
  uint64_t *accfull = empty + kStages;  // [2]
  uint64_t *accempty = accfull + 2;     // [2]
  uint64_t *drain = accempty + 2;       // the issuer's last commit: no MMA in flight at teardown
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int32_t *abort = reinterpret_cast<volatile int32_t *>(tmem_slot + 1);
  int32_t *pre = reinterpret_cast<int32_t *>(tmem_slot + 4);  // [E + 1]
  int32_t *cnt = pre + (p.E + 1);                             // [E]
  int32_t *tmp = cnt + p.E;                                   // [32]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;
  const int64_t K = p.K, N = p.N;
  const int CT = (int)((K + kBN - 1) / kBN);  // output column tiles
  const int nkp = (int)(N / kBK);             // reduction steps per projection
  const int nk = NPROJ * nkp;
  const int grows = p.group >= kBN ? 1 : kBN / p.group;  // group rows per coefficient tile
  const uint32_t stage_tx = kABytes + kPBytes + grows * (8 * 4 + kBK * 2);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&bready[s], kDqWarps);
      mbar_init(&empty[s], 1);
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
    cnt[e] = bad ? 0 : CT * ((b - a + kBM - 1) / kBM);
  }
  __syncthreads();
  block_exclusive_scan(cnt, E, pre, tmp);
  const int64_t total = pre[E];
  if ((int64_t)blockIdx.x >= total) return;

  auto tile_info = [&](int64_t tile) {
    BwdTile ti;
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
    // ---------------- producer
    if (lane == 0) {
      uint32_t it = 0;  // stages issued
      bool live = true;
      for (int64_t tile = blockIdx.x; tile < total && live; tile += gridDim.x) {
        const BwdTile ti = tile_info(tile);
        const int32_t row0 = (int32_t)(ti.r0 + (int64_t)ti.mt * kBM);
        const int64_t kk0 = (int64_t)ti.ct * kBN;
        const int32_t wrow = (int32_t)(ti.e * K + kk0);
        const int32_t grow = (int32_t)((ti.e * K + kk0) / p.group);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t s = it % kStages, use = it / kStages;
          if (use > 0 && !tc_wait(&empty[s], (use - 1) & 1, p.status, abort)) {
            live = false;
            break;
          }
          const int j = NPROJ == 2 ? kb / nkp : 0;
          const int32_t n0 = (kb - j * nkp) * kBK;
          uint8_t *st = stages + s * kStageBytes;
          uint8_t *cs = st + kABytes + kBBytes + kPBytes;
          mbar_arrive_expect_tx(&full[s], stage_tx);
          tma_load_2d(st, &maps.grad[j], &full[s], n0, row0);
          tma_load_2d(st + kABytes + kBBytes, &maps.qw[j], &full[s], n0 / 8, wrow);
          tma_load_2d(cs, &maps.qz[j], &full[s], n0 / 8, grow);
          tma_load_2d(cs + kZBytes, &maps.sc[j], &full[s], n0, grow);
        }
      }
      tma_drain(full, it, kStages, p.status);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t fmt = std::is_same<MT, __half>::value ? 0u : 1u;
      // D F32, A/B in the scale dtype, both K-major, N = 256, M = 128
      const uint32_t idesc =
          (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
      uint32_t it = 0, tcount = 0;
      bool live = true;
      for (int64_t tile = blockIdx.x; tile < total; tile += gridDim.x, ++tcount) {
        const uint32_t buf = tcount & 1, use = tcount >> 1;
        if (use > 0 && !tc_wait(&accempty[buf], (use - 1) & 1, p.status, abort)) break;
        tc_fence_after();
        const uint32_t dacc = tmem + buf * kBN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t s = it % kStages, ph = (it / kStages) & 1;
          if (!tc_wait(&full[s], ph, p.status, abort) || !tc_wait(&bready[s], ph, p.status, abort)) {
            live = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(stages + s * kStageBytes);
          const uint64_t adesc = smem_desc(a_addr, 16, 1024);
          const uint64_t bdesc = smem_desc(a_addr + kABytes, 16, 1024);
#pragma unroll
          for (int jj = 0; jj < kBK / 16; ++jj)
            umma_f16(dacc, adesc + (uint64_t)(2 * jj), bdesc + (uint64_t)(2 * jj), idesc, (kb | jj) != 0);
          umma_commit(&empty[s]);
        }
        if (!live) break;
        umma_commit(&accfull[buf]);
      }
      umma_commit(drain);  // arrives once every MMA issued above has completed
      mbar_wait(drain, 0, p.status);
    }
  } else if (warp < 2 + kDqWarps) {
    // ---------------- dequant warps: 256 coefficient rows x 8 words per step
    const int td = threadIdx.x - 64;  // 0..255
    const int wcol = td & 7;          // word column (8 reduction indices)
    const int rband = td >> 3;        // rows rband + 32 i, i = 0..7
    constexpr uint32_t M = Dq<MT>::kMagic2;
    const int b0 = (rband >> 3) * 1024 + (rband & 7) * 128 + ((wcol ^ (rband & 7)) << 4);
    uint32_t act_bad = 0;  // a converted input outside F16's normal range
    // gradients in the other 16-bit dtype are converted here unless a one-time copy was made
    const bool convert = !p.preconv && p.gdt != (std::is_same<MT, __half>::value ? MOE_F16 : MOE_BF16);
    // group row of band i = (32 i) / group; groups here are 64, 128 or >= 256 (one per tile)
    const int gshift = p.group >= kBN ? 8 : (p.group == 128 ? 7 : 6);
    uint32_t it = 0;
    bool live = true;
    for (int64_t tile = blockIdx.x; tile < total && live; tile += gridDim.x) {
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const uint32_t s = it % kStages, ph = (it / kStages) & 1;
        if (!tc_wait(&full[s], ph, p.status, abort)) {
          live = false;
          break;
        }
        uint8_t *st = stages + s * kStageBytes;
        if (convert) {
          uint4 *a4 = reinterpret_cast<uint4 *>(st);
#pragma unroll
          for (int i = 0; i < kABytes / 16 / 256; ++i) {
            uint4 v = a4[td + 256 * i];
            act_quad_to_mt<MT>(v, p.gdt, act_bad);
            a4[td + 256 * i] = v;
          }
        }
        const uint32_t *pk = reinterpret_cast<const uint32_t *>(st + kABytes + kBBytes) + rband * 8 + wcol;
        const uint8_t *cs = st + kABytes + kBBytes + kPBytes;
        const uint32_t *zs = reinterpret_cast<const uint32_t *>(cs) + wcol;
        const uint8_t *ss = cs + kZBytes + wcol * 16;
        uint8_t *bt = st + kABytes + b0;
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = pk[i * 32 * 8];
        uint32_t zp[4], sp[4];
        int cur = -1;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int gr = (32 * i) >> gshift;  // same for the whole warp
          if (gr != cur) {
            cur = gr;
            const uint32_t zw = zs[gr * 8];
            const uint4 sv = *reinterpret_cast<const uint4 *>(ss + gr * (kBK * 2));
            const uint32_t s4[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              zp[q] = nib_pair<M>(zw >> (4 * q));
              sp[q] = s4[q];
            }
          }
          uint4 c;
          c.x = Dq<MT>::coef(nib_pair<M>(w[i]), zp[0], sp[0]);        // n 0, 1
          c.y = Dq<MT>::coef(nib_pair<M>(w[i] >> 4), zp[1], sp[1]);   // n 2, 3
          c.z = Dq<MT>::coef(nib_pair<M>(w[i] >> 8), zp[2], sp[2]);   // n 4, 5
          c.w = Dq<MT>::coef(nib_pair<M>(w[i] >> 12), zp[3], sp[3]);  // n 6, 7
          *reinterpret_cast<uint4 *>(bt + i * 4096) = c;               // rows + 32
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bready[s]);
      }
    }
    if (act_bad) report(p.status, MOE_DEVICE_ERR_ACT_RANGE);
  } else {
    // ---------------- epilogue warps
    const int q = warp & 3;                     // TMEM lane quarter
    const int hf = (warp - 2 - kDqWarps) >> 2;  // column half drained by this warp
    const bool bf = p.odt == MOE_BF16;
    uint32_t tcount = 0;
    for (int64_t tile = blockIdx.x; tile < total; tile += gridDim.x, ++tcount) {
      const BwdTile ti = tile_info(tile);
      const uint32_t buf = tcount & 1;
      if (!tc_wait(&accfull[buf], (tcount >> 1) & 1, p.status, abort)) break;
      tc_fence_after();
      const int trow = ti.mt * kBM + 32 * q + lane;
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
      if (lane == 0) mbar_arrive(&accempty[buf]);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ------------------------------------------------------------------ launch

static size_t tcb_smem(int64_t E) {
  return 1024 + (size_t)tcb::kStages * tcb::kStageBytes + 256 + (size_t)(2 * E + 1 + 32) * 4;
}

// Whole 64-wide reduction steps, 16-column output chunks, and zero/scale
// groups that tile the 256-row coefficient tile evenly (at most 4 per tile).
bool tc_bwd_fits(const BwdParams &p) {
  const bool groups_ok = p.group % 64 == 0 && (tcb::kBN % p.group == 0 || p.group % tcb::kBN == 0);
  return p.N % tcb::kBK == 0 && p.K % 16 == 0 && groups_ok && tcb_smem(p.E) <= 227 * 1024;
}

template <typename MT, int NPROJ>
static moe_status launch_bwd_tc_t(const BwdParams &p, cudaStream_t st) {
  using namespace tcb;
  BwdMaps maps;
  const uint64_t NW = p.N / 8, rows = (uint64_t)p.E * p.K, grows_all = rows / p.group;
  const uint32_t gbox = p.group >= kBN ? 1 : kBN / p.group;
  for (int j = 0; j < 2; ++j) {
    const int jj = j < NPROJ ? j : 0;
    if (!make_map_2d(&maps.grad[j], p.grad[jj], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, p.N, p.A, kBK, kBM,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&maps.qw[j], p.qw[jj], CU_TENSOR_MAP_DATA_TYPE_INT32, 4, NW, rows, kBK / 8, kBN,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map_2d(&maps.qz[j], p.qz[jj], CU_TENSOR_MAP_DATA_TYPE_INT32, 4, NW, grows_all, kBK / 8, gbox,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map_2d(&maps.sc[j], p.sc[jj], CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, p.N, grows_all, kBK, gbox,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
      return set_error(MOE_ERR_CUDA, "tensor map encoding failed (tcgen05 input VJP)");
  }
  const size_t smem = tcb_smem(p.E);
  auto kern = awq_bwd_tc_kernel<MT, NPROJ>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  kern<<<num_sms(), kThreads, smem, st>>>(maps, p);
  return check_launch("awq_bwd_tc_kernel");
}

moe_status launch_bwd_tc(const BwdParams &p, int nproj, bool bf16_mma, cudaStream_t st) {
  if (bf16_mma) return nproj == 2 ? launch_bwd_tc_t<__nv_bfloat16, 2>(p, st) : launch_bwd_tc_t<__nv_bfloat16, 1>(p, st);
  return nproj == 2 ? launch_bwd_tc_t<__half, 2>(p, st) : launch_bwd_tc_t<__half, 1>(p, st);
}

}  // namespace moe
