// Grouped AWQ forward for small per-expert batches (decode): packed words
// stream through shared memory by TMA and warp-level tensor-core tiles
// (mma.sync m16n8k16, FP32 accumulate) consume them.  Here the packed-weight
// bytes bound the time, so the design is about reading each weight byte
// exactly once, in whole 128-byte lines, with enough bytes in flight.
//
// ruda-tensor 0.21.34, src/packed_experts.rs -- packed_expert_forward /
//   packed_swiglu_forward (gate/up/down of the selected experts, SwiGLU);
// ruda-tensor 0.21.33, src/frozen_awq.rs -- AWQ nibble order and scale-dtype
//   coefficient rounding.
//
// Work item = (expert e, token tile tt of 8*NT rows, slab sl).  A slab is
// 512 output columns: for the gate/up pair, 32 packed word columns (one
// 128-byte row segment) of each projection; for a single projection, 64 word
// columns (two 128-byte segments).  An item is K/ROWS pipeline stages of
// ROWS input rows (32, 64 or 128, the largest the group size allows).  The
// stages of all items, expert-major, form one list that the persistent CTAs
// (8 warps; 2 per SM) split into equal contiguous ranges (stream-K), so
// every CTA streams the same number of weight bytes whatever the routing.
//   copies: per stage two TMA boxes of [ROWS rows][32 words] with 128-byte
//     swizzle into a ring (64 KB in flight for 128-row stages), each issued
//     once every warp released the ring slot's previous stage, by lane 0 of
//     the warps in turn (stage r by warp r mod 8, so no warp carries all the
//     issue work); per 512 input rows of an item, 1-D bulk copies of the
//     item's activation rows (lane 0 of warp 0; double-buffered, one chunk
//     ahead).
//   warp w: box w/4, word columns (w%4)*8 .. +7 of it, all rows of the
//     stage.  Lane (g, t) reads rows t, t+4, t+8, t+12 of column g (the
//     MMA's K index {2t, 2t+1, 2t+8, 2t+9} stands for them); the swizzle
//     keeps those reads at most 2-way bank-conflicted.  Each activation
//     chunk is converted to the scale dtype and permuted to that row order
//     once, so each B fragment is one 8-byte shared load.
//   end of a CTA's part of an item: a CTA that holds the whole item sends
//     the accumulators through shared memory to bias, rounding and SwiGLU;
//     CTAs sharing an item store FP32 partial sums, and a second kernel adds
//     the parts in part order (deterministic) and finishes the rows.
#include <cudaTypedefs.h>

#include <mutex>

#include "dequant.cuh"
#include "proj.cuh"
#include "tma.cuh"

namespace moe {

// ------------------------------------------------------------------ host: tensor maps

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_map_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dt, int elem_bytes, uint64_t inner,
                 uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ device

namespace stream {
constexpr int kCW = 8;                    // consumer warps
constexpr int kThreads = kCW * 32;  // lane 0 of warp 0 also issues the copies
constexpr int kBoxW = 32;                 // words per box row (128 bytes)
constexpr int kF = 512;                   // output columns of a unit
constexpr int kBarBytes = 1024;           // barrier block; stages start 1024-byte aligned
// A stage is ROWS input rows (ROWS / 16 MMA steps) of two [ROWS][32-word]
// boxes; deeper stages spread the per-stage bookkeeping over more weight
// bytes (a 128-row stage is 32 KB, so two of them keep 64 KB in flight).
template <int ROWS>
struct Geo {
  static constexpr int kRows = ROWS;
  static constexpr int kBox = ROWS * kBoxW * 4;
  static constexpr int kStageBytes = 2 * kBox;
  static constexpr int kStages = ROWS == 128 ? 2 : ROWS == 64 ? 4 : 6;  // 64 / 64 / 48 KB in flight per CTA
};
}  // namespace stream

// Largest e with pre[e] <= u (pre is the exclusive prefix of units per expert).
__device__ __forceinline__ int unit_expert(const int32_t *pre, int E, int64_t u) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= u) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Byte offset of word (row, col) in a [32][32]-word box written by TMA with
// 128-byte swizzle (16-byte chunk index XOR row mod 8).
__device__ __forceinline__ int box_offset(int row, int col) {
  return row * 128 + ((((col >> 2) ^ row) & 7) << 4) + ((col & 3) << 2);
}

// ------------------------------------------------------------------ stream-K schedule
//
// Work item = (expert e, token tile tt of 8*NT rows, slab sl), expert-major;
// an item is nst = K / ROWS pipeline stages.  The stages of all items form
// one list that the CTAs split evenly (each takes a contiguous range of at
// least kMinStages stages), so a CTA may start or end inside an item.  A CTA
// that holds a whole item finishes its rows in the fused epilogue; the CTAs
// that share an item store their FP32 partial sums in part order (part =
// the CTA's rank among them) and a second kernel adds the parts in that
// order (deterministic) and finishes the rows.
constexpr int kMinStages = 4;

__host__ __device__ __forceinline__ int64_t sk_grid(int64_t G, int64_t grid) {
  int64_t g = G / kMinStages;
  if (g > grid) g = grid;
  return g < 1 ? 1 : g;
}
// CTA holding stage s when G stages are split over `grid` CTAs.
__device__ __forceinline__ int64_t sk_owner(int64_t s, int64_t G, int64_t grid) {
  return ((s + 1) * grid + G - 1) / G - 1;
}
// Parts an item of nst stages can be split into (host bound of the workspace).
__host__ __device__ __forceinline__ int sk_max_parts(int nst) { return (nst - 1 + kMinStages - 1) / kMinStages + 1; }

struct ItemInfo {
  int e, tt, sl;
  int64_t r0;
  int m;
};

__device__ __forceinline__ ItemInfo item_info(const int32_t *pre, const int32_t *offsets, int E, int S, int64_t i) {
  ItemInfo ii;
  ii.e = unit_expert(pre, E, i);
  const int local = (int)(i - pre[ii.e]);  // item counts fit 32 bits (pre is int32)
  ii.tt = local / S;
  ii.sl = local - ii.tt * S;
  ii.r0 = offsets[ii.e];
  ii.m = offsets[ii.e + 1] - (int32_t)ii.r0;
  return ii;
}

template <typename MT, int NPROJ, int NT, int ROWS>
__global__ void __launch_bounds__(stream::kThreads, 2)
    awq_fwd_stream_kernel(const __grid_constant__ CUtensorMap map0, const __grid_constant__ CUtensorMap map1,
                          ProjParams p) {
  pdl_enter();  // programmatic dependent launch: the previous kernel is done
  using namespace stream;
  constexpr int kRows = Geo<ROWS>::kRows, kBox = Geo<ROWS>::kBox, kStageBytes = Geo<ROWS>::kStageBytes;
  constexpr int kStages = Geo<ROWS>::kStages;
  constexpr int kSteps = ROWS / 16;
  constexpr int kXst = 512 / ROWS;        // stages per activation chunk
  constexpr int kXRows = kXst * ROWS;     // input rows per activation chunk (512)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 128-byte-swizzled TMA boxes need 1024-byte aligned destinations
  uint8_t *smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int E = p.E;
  const int64_t K = p.K;
  const int64_t NW = p.N / 8;
  constexpr int kSlabW = NPROJ == 2 ? kBoxW : 2 * kBoxW;  // word columns of a slab
  const int S = (int)((NW + kSlabW - 1) / kSlabW);       // slabs per expert
  const int nst = (int)(K / kRows);                      // stages per item
  constexpr int xs_pitch = kXRows * 2 + 16;  // bytes per converted token row (pad: conflict-free B loads)
  constexpr int xraw_bytes = 8 * NT * kXRows * 2;
  const int64_t ncols = (int64_t)NPROJ * p.N;  // columns of the partial rows

  uint64_t *full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *empty = full + kStages;
  uint64_t *xfull = empty + kStages;
  uint64_t *xempty = xfull + 2;
  uint8_t *stages = smem + kBarBytes;
  uint8_t *xraw = stages + kStages * kStageBytes;  // 2 buffers
  uint8_t *xs = xraw + 2 * xraw_bytes;
  float *red = reinterpret_cast<float *>(xs + 8 * NT * xs_pitch);  // [8*NT][kF]
  int32_t *pre = reinterpret_cast<int32_t *>(red + 8 * NT * kF);    // [E + 1]
  int32_t *cnt = pre + (E + 1);                                    // [E]
  int32_t *tmp = cnt + E;                                          // [32]
  int32_t *issued_hi = tmp + 32;                                   // [1]: stages issued (relative), max
  volatile int32_t *abort = reinterpret_cast<volatile int32_t *>(xempty + 2);
#ifdef MOE_TEST_HOOKS
  uint64_t *stall = xempty + 3;  // test build only: a barrier nothing arrives on
#endif

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&xfull[b], 1);
      mbar_init(&xempty[b], kCW);
    }
    *abort = 0;
#ifdef MOE_TEST_HOOKS
    mbar_init(stall, 1);
#endif
    fence_mbar_init();
  }
  // items per expert; an inconsistent row range is flagged and skipped
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int32_t a = p.offsets[e], b = p.offsets[e + 1];
    const bool bad = a < 0 || b < a || (int64_t)b > p.A || (e == 0 && a != 0) || (e == E - 1 && (int64_t)b != p.A);
    if (bad && blockIdx.x == 0) report(p.status, MOE_DEVICE_ERR_OFFSETS);
    cnt[e] = bad ? 0 : S * ((b - a + 8 * NT - 1) / (8 * NT));
  }
  __syncthreads();
  block_exclusive_scan(cnt, E, pre, tmp);
  // the reduction kernel reads the item prefix from the workspace
  if (blockIdx.x == 0 && p.counters)
    for (int e = threadIdx.x; e <= E; e += blockDim.x) p.counters[e] = pre[e];
  const int64_t G = (int64_t)pre[E] * nst;
  const int64_t grid = sk_grid(G, gridDim.x);
  if ((int64_t)blockIdx.x >= grid) return;  // nothing issued, nothing waited for
  const int64_t g0 = G * blockIdx.x / grid, g1 = G * (blockIdx.x + 1) / grid;

  // ---------------- copies, issued by lane 0 of consumer warp 0: stage
  // j - g0 of the ring is stage j of the list, issued once all consumers
  // released the slot's previous stage; activation chunks one ahead.
  int64_t nxt = g0;        // next stage to issue (thread 0 only)
  uint32_t xissued = 0;    // activation chunks issued (thread 0 only)
  bool plive = true;       // thread 0 stops issuing after a failed wait
  const bool issuer = threadIdx.x == 0;
  int64_t iss_i = -1;
  ItemInfo iss_ii{};
  auto issue_info = [&](int64_t i) -> const ItemInfo & {
    if (i != iss_i) {
      iss_i = i;
      iss_ii = item_info(pre, p.offsets, E, S, i);
    }
    return iss_ii;
  };
  // activation chunk of stage j (rows of j's item, the 512 input rows holding j)
  auto load_x = [&](int64_t j, uint32_t xi) {
    const int64_t i = j / nst;
    const int ch = (int)(j - i * nst) / kXst;
    const ItemInfo &ii = issue_info(i);
    const int tok0 = ii.tt * 8 * NT, mrows = min(8 * NT, ii.m - tok0);
    const int64_t k0 = (int64_t)ch * kXRows;
    const int64_t len = min((int64_t)kXRows, K - k0);
    const uint32_t xb = xi & 1, xuse = xi >> 1;
    if (xuse > 0 && !tc_wait(&xempty[xb], (xuse - 1) & 1, p.status, abort)) {
      plive = false;
      return;
    }
    mbar_arrive_expect_tx(&xfull[xb], (uint32_t)(mrows * len * 2));
    for (int r = 0; r < mrows; ++r)
      bulk_load(xraw + xb * xraw_bytes + r * kXRows * 2, p.x + act_row(p, ii.r0 + tok0 + r) * K + k0,
                (uint32_t)(len * 2), &xfull[xb]);
    ++xissued;
  };
  auto issue_stage_ic = [&](int64_t j, int64_t i, int c) {
    const uint32_t s = (uint32_t)((j - g0) % kStages);
    const ItemInfo &ii = issue_info(i);
    const int32_t row0 = (int32_t)(ii.e * K + (int64_t)c * kRows);
    mbar_arrive_expect_tx(&full[s], kStageBytes);
    uint8_t *dst = stages + s * kStageBytes;
    if (NPROJ == 2) {
      tma_load_2d(dst, &map0, &full[s], ii.sl * kBoxW, row0);
      tma_load_2d(dst + kBox, &map1, &full[s], ii.sl * kBoxW, row0);
    } else {
      tma_load_2d(dst, &map0, &full[s], ii.sl * 2 * kBoxW, row0);
      tma_load_2d(dst + kBox, &map0, &full[s], ii.sl * 2 * kBoxW + kBoxW, row0);
    }
  };
  auto issue_stage = [&](int64_t j) {
    const int64_t i = j / nst;
    issue_stage_ic(j, i, (int)(j - i * nst));
  };
  // blocking: issue every stage up to `upto` (waits for the slots' release)
  auto issue_upto = [&](int64_t upto) {
    while (plive && nxt <= upto && nxt < g1) {
      const uint32_t s = (uint32_t)((nxt - g0) % kStages), use = (uint32_t)((nxt - g0) / kStages);
      if (use > 0 && !tc_wait(&empty[s], (use - 1) & 1, p.status, abort)) {
        plive = false;
        break;
      }
      issue_stage(nxt++);
    }
  };
  if (issuer && g0 < g1) {
    load_x(g0, 0);
    issue_upto(g0 + kStages - 1);
    *issued_hi = (int32_t)(nxt - g0);
  }
  // Stages past the first kStages rotate over the warps: stage g0 + r (r >=
  // kStages) is issued by lane 0 of warp r % kCW at the top of iteration
  // g0 + r - kStages + 1, once every warp released the slot's previous
  // stage, so no single warp carries the issue work.
  bool rlive = true;
  auto issue_rotating = [&](int64_t j, int64_t i, int c) {
    const int64_t st = j + kStages - 1;  // the stage due now
    const int64_t r = st - g0;
    if (r < kStages || st >= g1 || !rlive || lane != 0 || (int)(r % kCW) != warp) return;
    const uint32_t s = (uint32_t)(r % kStages), use = (uint32_t)(r / kStages);
    if (!tc_wait(&empty[s], (use - 1) & 1, p.status, abort)) {
      rlive = false;
      return;
    }
    c += kStages - 1;  // item and stage of st
    while (c >= nst) {
      c -= nst;
      ++i;
    }
    issue_stage_ic(st, i, c);
    atomicMax(issued_hi, (int32_t)(r + 1));
  };

  // ---------------- consumers
  uint32_t act_bad = 0;  // a converted input outside F16's normal range
  const int g = lane >> 2, t = lane & 3;
  const int bw = warp >> 2, cgw = warp & 3;  // box and column group of this warp
  const int jw = NPROJ == 2 ? bw : 0;        // projection of this warp
  const int64_t ngroups = K / p.group;
  const int32_t *qz = p.qz[jw];
  const uint16_t *sc = p.sc[jw];
  // byte offsets of rows t and t+4 of column cgw*8+g in a swizzled box; rows
  // t + 4i + 16h differ from these by multiples of 8 rows (same swizzle)
  const int woff0 = box_offset(t, cgw * 8 + g), woff1 = box_offset(t + 4, cgw * 8 + g);
  const int spg = p.group / kRows;  // stages per group (group % kRows == 0 on this path)

  float acc[NT][4][4];
  FwdConsts<MT> cst;
  ItemInfo ii{};
  int tok0 = 0, mrows = 0, seg_c0 = 0, seg_c1 = 0, xbase = 0, gstage = 0;
  int64_t wc = 0, grp = 0;
  bool wc_ok = false;
  const int32_t *qzp = qz;
  const uint16_t *scp = sc;
  uint32_t pf_zw = 0u;
  uint4 pf_sv = make_uint4(0, 0, 0, 0);
  uint32_t it = 0, xi = 0;
  // item i and stage c of stage j, advanced without a division
  int64_t i = g0 / nst;
  int c = (int)(g0 - i * nst);
  for (int64_t j = g0; j < g1; ++j, ++it, c = (c + 1 == nst) ? (++i, 0) : c + 1) {
    if (j == g0 || c == 0) {  // a segment of item i starts: its rows, columns and first group
      ii = item_info(pre, p.offsets, E, S, i);
      tok0 = ii.tt * 8 * NT;
      mrows = min(8 * NT, ii.m - tok0);
      seg_c0 = c;
      seg_c1 = (int)min((int64_t)nst, (int64_t)c + (g1 - j));
      wc = NPROJ == 2 ? (int64_t)ii.sl * kBoxW + cgw * 8 + g : (int64_t)ii.sl * 2 * kBoxW + bw * kBoxW + cgw * 8 + g;
      wc_ok = wc < NW;
      const int64_t wcs = wc_ok ? wc : 0;
      qzp = qz + ((int64_t)ii.e * ngroups) * NW + wcs;
      scp = sc + ((int64_t)ii.e * ngroups) * p.N + 8 * wcs;
      grp = (int64_t)c * kRows / p.group;
      gstage = (int)(((int64_t)c * kRows % p.group) / kRows);
      pf_zw = wc_ok ? (uint32_t)__ldg(qzp + grp * NW) : 0u;
      pf_sv = wc_ok ? __ldg(reinterpret_cast<const uint4 *>(scp + grp * p.N)) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[nt][q][k] = 0.f;
      }
    }
    if (j == g0 || c % kXst == 0) {
      // a new activation chunk: request the next one, then convert this one
      // (raw rows -> scale dtype, row order t, t+4, t+8, t+12 per 16).  After
      // an abort every consumer warp still runs the loop (the named barriers
      // stay matched) but waits for, computes and arrives on nothing.
      const uint32_t xcur = xi++;
      xbase = c - c % kXst;
      if (issuer && plive) {
        const int64_t nc = (int64_t)xbase + kXst;
        const int64_t jn = nc < nst ? i * nst + nc : (i + 1) * nst;
        if (jn < g1) load_x(jn, xcur + 1);
      }
      const uint32_t xb = xcur & 1;
      // every consumer is done reading the previous chunk's converted tile
      named_barrier(1, kCW * 32);
      const bool xok = tc_wait(&xfull[xb], (xcur >> 1) & 1, p.status, abort);
      if (xok) {
        const uint8_t *src = xraw + xb * xraw_bytes;
        const int len = (int)min((int64_t)kXRows, K - (int64_t)xbase * kRows);
        const int per_tok = len / 8, halves = mrows * per_tok;
        const bool whole = per_tok == kXRows / 8;
        for (int q = threadIdx.x; q < halves; q += kCW * 32) {
          const int tok = whole ? q / (kXRows / 8) : q / per_tok;
          const int hb = q - tok * per_tok, blk = hb >> 1, h = hb & 1;
          const uint4 v = *reinterpret_cast<const uint4 *>(src + (tok * kXRows + blk * 16 + h * 8) * 2);
          uint32_t pr[4] = {prmt(v.x, v.z, 0x5410u), prmt(v.x, v.z, 0x7632u), prmt(v.y, v.w, 0x5410u),
                            prmt(v.y, v.w, 0x7632u)};  // (row i, row i+4) of the half
          act_pairs_to_mt<MT, 4>(pr, p.act_dt, act_bad);
          uint8_t *dst = xs + tok * xs_pitch + (blk * 16 + 2 * h) * 2;
#pragma unroll
          for (int k = 0; k < 4; ++k) *reinterpret_cast<uint32_t *>(dst + 8 * k) = pr[k];
        }
      }
      __syncwarp();
      if (lane == 0 && xok) mbar_arrive(&xempty[xb]);
      named_barrier(1, kCW * 32);
    }
    const uint32_t s = (uint32_t)((j - g0) % kStages), ph = (uint32_t)(((j - g0) / kStages) & 1);
    if (gstage == 0 || j == g0 || c == seg_c0) {  // a stage lies inside one group
      load_consts_fast<MT>(cst, pf_zw, pf_sv);
      if (wc_ok && (grp + 1) * p.group < K) {  // prefetch the next group
        pf_zw = (uint32_t)__ldg(qzp + (grp + 1) * NW);
        pf_sv = __ldg(reinterpret_cast<const uint4 *>(scp + (grp + 1) * p.N));
      }
    }
    if (++gstage == spg) {
      gstage = 0;
      ++grp;
    }
    issue_rotating(j, i, c);
    // warp-uniform: the MMAs below are warp-wide
    const bool sok = __all_sync(0xffffffffu, tc_wait(&full[s], ph, p.status, abort));
    if (sok) {
      const uint8_t *box0 = stages + s * kStageBytes + bw * kBox;
      // two 16-row steps at a time keep the register footprint of a 32-row stage
#pragma unroll 1
      for (int hh = 0; hh < kSteps; hh += 2) {
        const uint8_t *box = box0 + (16 * hh) * 128;
        const int xrow0 = kRows * (c - xbase) + 16 * hh;
        uint32_t w[2][4];
        uint32_t b0[2][NT], b1[2][NT];
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // 16-row steps: rows 16h + {t, t+4, t+8, t+12}
          w[h][0] = *reinterpret_cast<const uint32_t *>(box + woff0 + (16 * h) * 128);
          w[h][1] = *reinterpret_cast<const uint32_t *>(box + woff1 + (16 * h) * 128);
          w[h][2] = *reinterpret_cast<const uint32_t *>(box + woff0 + (16 * h + 8) * 128);
          w[h][3] = *reinterpret_cast<const uint32_t *>(box + woff1 + (16 * h + 8) * 128);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const uint2 bv =
                *reinterpret_cast<const uint2 *>(xs + (nt * 8 + g) * xs_pitch + (xrow0 + 16 * h + 4 * t) * 2);
            b0[h][nt] = bv.x;
            b1[h][nt] = bv.y;
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t af[4][4];
          fwd_step<MT>(w[h][0], w[h][1], w[h][2], w[h][3], cst, af);
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma16816<MT>(acc[nt][q], af[q], b0[h][nt], b1[h][nt]);
        }
      }
    }
    __syncwarp();
    if (lane == 0 && sok) mbar_arrive(&empty[s]);
    if (c != seg_c1 - 1) continue;

    // ---------------- the segment ends here
    const bool seg_ok = !*abort;  // no stores from a segment an abort cut short
    if (seg_c0 != 0 || seg_c1 != nst) {
      // a part of a shared item: FP32 partial sums to partials[part][row][column]
      const int64_t part = (int64_t)blockIdx.x - sk_owner(i * nst, G, grid);
      float *prow = p.partials + (part * p.A + ii.r0 + tok0) * ncols;
      if (wc_ok && seg_ok) {
        const int64_t col0 = (int64_t)jw * p.N + wc * 8;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int d = 0; d < 2; ++d) {
            const int tk = nt * 8 + 2 * t + d;
            if (tk < mrows) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                __stcg(reinterpret_cast<float2 *>(prow + tk * ncols + col0 + 2 * q),
                       make_float2(acc[nt][q][d], acc[nt][q][2 + d]));
            }
          }
      }
      continue;
    }
    // the whole item in this CTA: accumulators -> red[token][column], epilogue
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int f = bw * 256 + cgw * 64 + 8 * g + 2 * q, tk = nt * 8 + 2 * t;
        red[tk * kF + f] = acc[nt][q][0];
        red[(tk + 1) * kF + f] = acc[nt][q][1];
        red[tk * kF + f + 1] = acc[nt][q][2];
        red[(tk + 1) * kF + f + 1] = acc[nt][q][3];
      }
    named_barrier(1, kCW * 32);
    constexpr int kOut = NPROJ == 2 ? kF / 2 : kF;  // output columns of the item
    for (int v8 = threadIdx.x; v8 < mrows * (kOut / 8); v8 += kCW * 32) {
      const int tk = v8 / (kOut / 8), fq = (v8 % (kOut / 8)) * 8;
      const int64_t n0 = (int64_t)ii.sl * kOut + fq;
      if (n0 >= p.N || !seg_ok) continue;
      const float *g8 = red + tk * kF + fq;
      finish8<NPROJ>(p, ii.e, ii.r0 + tok0 + tk, n0, g8, g8 + 256);
    }
    named_barrier(1, kCW * 32);  // red is free again
  }
  // nothing asynchronous may be in flight at exit (abort protocol): every
  // warp's issues are done once all warps left the loop
  named_barrier(1, kCW * 32);
  if (issuer) {
    tma_drain(full, (uint32_t)*(volatile int32_t *)issued_hi, kStages, p.status);
    tma_drain(xfull, xissued, 2, p.status);
  }
  if (act_bad) report(p.status, MOE_DEVICE_ERR_ACT_RANGE);
#ifdef MOE_TEST_HOOKS
  // Test build only: one consumer thread waits, after every stage and
  // activation tile of its CTA has landed (each was waited for above), on a
  // phase that nothing completes, with a 1 ms limit, so a test can watch a
  // bounded wait give up and report MOE_DEVICE_ERR_TIMEOUT.
  if (p.test_stall && warp == 0 && lane == 0) {
    const uint64_t t0 = global_ns();
    bool done = false;
    while (!done && global_ns() - t0 < 1000000ull) done = mbar_try_wait(stall, 0);
    if (!done) report(p.status, MOE_DEVICE_ERR_TIMEOUT);
  }
#endif
}

// Items split over several CTAs: out[r, n..n+8) from the sum of their parts
// (in part order), then bias, rounding and SwiGLU as in the fused epilogue.
// p.counters holds the item prefix per expert, p.kq the first kernel's grid.
template <int NPROJ, int NT, int ROWS>
__global__ void __launch_bounds__(256) awq_stream_reduce_kernel(ProjParams p) {
  pdl_enter();  // programmatic dependent launch: the previous kernel is done
  using namespace stream;
  constexpr int kSlabW = NPROJ == 2 ? kBoxW : 2 * kBoxW;
  constexpr int kOut = kSlabW * 8;
  const int64_t ncols = (int64_t)NPROJ * p.N;
  const int64_t per_row = p.N / 8;
  const int64_t total = p.A * per_row;
  const int S = (int)((p.N / 8 + kSlabW - 1) / kSlabW);
  const int nst = (int)(p.K / ROWS);
  // the row offsets and item prefix in shared memory: the searches below
  // then cost no global round trips
  extern __shared__ int32_t rsm[];
  int32_t *off_s = rsm, *pre_s = rsm + (p.E + 1);
  for (int e = threadIdx.x; e <= p.E; e += blockDim.x) {
    off_s[e] = p.offsets[e];
    pre_s[e] = p.counters[e];
  }
  __syncthreads();
  const int64_t G = (int64_t)pre_s[p.E] * nst;
  const int64_t grid = sk_grid(G, p.kq);
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < total; v += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = v / per_row, n0 = (v % per_row) * 8;
    // expert of row r: largest e with offsets[e] <= r (non-empty range)
    int lo = 0, hi = p.E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (off_s[mid] <= r) lo = mid;
      else hi = mid - 1;
    }
    const int64_t tt = (r - off_s[lo]) / (8 * NT);
    const int64_t item = pre_s[lo] + tt * S + n0 / kOut;
    if (r < off_s[lo] || item < 0 || item >= pre_s[p.E]) continue;  // rows of a range flagged bad
    const int64_t first = sk_owner(item * nst, G, grid), last = sk_owner(item * nst + nst - 1, G, grid);
    if (first == last || last - first >= sk_max_parts(nst)) continue;  // the fused epilogue wrote these outputs
    float a[NPROJ][8];
#pragma unroll
    for (int jj = 0; jj < NPROJ; ++jj)
#pragma unroll
      for (int k = 0; k < 8; ++k) a[jj][k] = 0.f;
    for (int64_t part = 0; part <= last - first; ++part) {
      const float *src = p.partials + (part * p.A + r) * ncols + n0;
#pragma unroll
      for (int jj = 0; jj < NPROJ; ++jj) {
        const float4 x0 = __ldcg(reinterpret_cast<const float4 *>(src + jj * p.N));
        const float4 x1 = __ldcg(reinterpret_cast<const float4 *>(src + jj * p.N + 4));
        a[jj][0] += x0.x; a[jj][1] += x0.y; a[jj][2] += x0.z; a[jj][3] += x0.w;
        a[jj][4] += x1.x; a[jj][5] += x1.y; a[jj][6] += x1.z; a[jj][7] += x1.w;
      }
    }
    finish8<NPROJ>(p, lo, r, n0, a[0], a[NPROJ - 1]);
  }
}

// ------------------------------------------------------------------ launch

static size_t stream_smem(int nt, int64_t E, int rows) {
  using namespace stream;
  const size_t ring = rows == 128  ? (size_t)Geo<128>::kStages * Geo<128>::kStageBytes
                     : rows == 64 ? (size_t)Geo<64>::kStages * Geo<64>::kStageBytes
                                  : (size_t)Geo<32>::kStages * Geo<32>::kStageBytes;
  return 1024 /* alignment slack */ + kBarBytes + ring + 2 * (size_t)8 * nt * 512 * 2 +
         (size_t)8 * nt * (512 * 2 + 16) + (size_t)8 * nt * kF * 4 + (size_t)(2 * E + 1 + 32 + 4) * 4;
}

// Workspace: the parts of split items (at most sk_max_parts per item) and
// the item prefix for the reduction.
StreamPlan stream_plan(int64_t A, int64_t K, int64_t N, int64_t E, int64_t group, int nproj, int nt) {
  StreamPlan pl{};
  pl.fits = false;
  // TMA needs 16-byte word-row pitches; a stage lies inside one group
  if (N % 32 != 0 || K % 32 != 0 || group % 32 != 0) return pl;
  const int rows = (K % 128 == 0 && group % 128 == 0) ? 128 : (K % 64 == 0 && group % 64 == 0) ? 64 : 32;
  const int parts = sk_max_parts((int)(K / rows));
  const size_t pbytes = (size_t)parts * A * nproj * N * 4;
  if (pbytes > ((size_t)512 << 20)) return pl;
  if (stream_smem(nt, E, rows) > 200 * 1024) return pl;
  pl.rows = rows;
  pl.fits = true;
  pl.kq = parts;
  pl.partial_off = 0;
  pl.counter_off = (pbytes + 255) & ~size_t(255);
  pl.bytes = pl.counter_off + (size_t)(E + 1) * 4;
  return pl;
}

#ifdef MOE_TEST_HOOKS
// Test build only: arms the stall of the next streaming-tile launches.
static int g_test_stall = 0;
extern "C" __attribute__((visibility("default"))) int32_t moe_test_arm_stall(int32_t on) {
  const int prev = g_test_stall;
  g_test_stall = on ? 1 : 0;
  return prev;
}
#endif

template <typename MT, int NPROJ, int NT, int ROWS>
static moe_status launch_stream_r(const ProjParams &p0, cudaStream_t st) {
  ProjParams p = p0;
#ifdef MOE_TEST_HOOKS
  p.test_stall = g_test_stall;
#endif
  using namespace stream;
  constexpr int kRows = Geo<ROWS>::kRows;
  CUtensorMap m0, m1;
  const uint64_t NW = p.N / 8, rows = (uint64_t)p.E * p.K;
  if (!make_map_2d(&m0, p.qw[0], CU_TENSOR_MAP_DATA_TYPE_INT32, 4, NW, rows, kBoxW, kRows,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&m1, p.qw[NPROJ - 1], CU_TENSOR_MAP_DATA_TYPE_INT32, 4, NW, rows, kBoxW, kRows,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return set_error(MOE_ERR_CUDA, "tensor map encoding failed for the packed words");
  const size_t smem = stream_smem(NT, p.E, ROWS);
  auto kern = awq_fwd_stream_kernel<MT, NPROJ, NT, ROWS>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const int grid = num_sms() * (smem <= 110 * 1024 ? 2 : 1);
  p.kq = grid;
  launch_pdl(kern, dim3(grid), dim3(kThreads), smem, st, m0, m1, p);
  moe_status s = check_launch("awq_fwd_stream_kernel");
  if (s != MOE_OK) return s;
  const int64_t work = p.A * (p.N / 8);
  int64_t blocks = (work + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  launch_pdl(awq_stream_reduce_kernel<NPROJ, NT, ROWS>, dim3((unsigned)blocks), dim3(256),
             (size_t)(2 * (p.E + 1)) * sizeof(int32_t), st, p);
  return check_launch("awq_stream_reduce_kernel");
}

template <typename MT, int NPROJ, int NT>
static moe_status launch_stream_t(const ProjParams &p, int rows, cudaStream_t st) {
  if (rows == 128) return launch_stream_r<MT, NPROJ, NT, 128>(p, st);
  return rows == 64 ? launch_stream_r<MT, NPROJ, NT, 64>(p, st) : launch_stream_r<MT, NPROJ, NT, 32>(p, st);
}

moe_status launch_fwd_stream(ProjParams p, int nproj, bool bf16_mma, int nt, void *ws, size_t ws_bytes,
                             cudaStream_t st) {
  const StreamPlan pl = stream_plan(p.A, p.K, p.N, p.E, p.group, nproj, nt);
  if (!ws || ws_bytes < pl.bytes || !aligned16(ws))
    return set_error(MOE_ERR_WORKSPACE, "projection workspace of %zu bytes, need %zu (16-byte aligned)", ws_bytes,
                     pl.bytes);
  p.partials = reinterpret_cast<float *>(static_cast<char *>(ws) + pl.partial_off);
  p.counters = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + pl.counter_off);
  const int r = pl.rows;
  if (bf16_mma) {
    if (nproj == 2)
      return nt == 2 ? launch_stream_t<__nv_bfloat16, 2, 2>(p, r, st) : launch_stream_t<__nv_bfloat16, 2, 1>(p, r, st);
    return nt == 2 ? launch_stream_t<__nv_bfloat16, 1, 2>(p, r, st) : launch_stream_t<__nv_bfloat16, 1, 1>(p, r, st);
  }
  if (nproj == 2) return nt == 2 ? launch_stream_t<__half, 2, 2>(p, r, st) : launch_stream_t<__half, 2, 1>(p, r, st);
  return nt == 2 ? launch_stream_t<__half, 1, 2>(p, r, st) : launch_stream_t<__half, 1, 1>(p, r, st);
}

}  // namespace moe
