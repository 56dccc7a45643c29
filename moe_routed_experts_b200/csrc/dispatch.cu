// Top-k routing and stable expert-sorted COPY dispatch.
//
// ruda-tensor 0.21.38, src/moe_exchange.rs -- MoeDispatchOps::moe_dispatch:
// selection and FP32 continuous weights, then a device COPY of each selected
// row into an expert-sorted buffer whose U32 row_experts ascend.
//
// Three launches (two when the tokens fit one chunk):
//   1. route_rank: one warp per token selects its top-k experts and their
//      weights; per chunk of tokens, one warp assigns each (token, j) its
//      rank among the chunk's rows of the same expert in token order
//      (__match_any_sync groups equal experts; lanes are ordered by token),
//      and the chunk histogram is written.  A single chunk also scans its
//      histogram into the expert offsets.
//   2. scan: per expert, an exclusive scan of the chunk histograms in chunk
//      order (the chunk bases) and of the totals in expert order (offsets).
//   3. scatter: row = offsets[e] + chunk_base[chunk][e] + rank; writes the
//      row maps and copies the activation rows, spread over warps in
//      512-byte segments.
// Row order is (expert, token) by construction, with no atomics whose order
// could vary between runs.
#include <math.h>

#include "common.cuh"

namespace moe {

constexpr int kScanThreads = 1024;
constexpr int kMaxChunks = 1024;

// Tokens per chunk: 64 (the ranks come from one 64-bit token mask per
// expert), or a larger power of two keeping the chunk count <= kMaxChunks
// (ranked by one warp in token order).
static int64_t route_chunk(int64_t T) {
  int64_t c = 64;
  while ((T + c - 1) / c > kMaxChunks) c *= 2;
  return c;
}

static int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

struct RouteWs {
  int64_t chunk, nchunks;
  size_t hist_off, rank_off, bytes;
};

static RouteWs route_ws_layout(int64_t T, int64_t E, int32_t k) {
  RouteWs w;
  w.chunk = route_chunk(T > 0 ? T : 1);
  w.nchunks = (T + w.chunk - 1) / w.chunk;
  if (w.nchunks < 1) w.nchunks = 1;
  w.hist_off = 0;
  w.rank_off = (size_t)round_up(w.nchunks * E * 4, 256);
  w.bytes = w.rank_off + (size_t)round_up(T * (int64_t)k * 4, 256);
  if (w.bytes < 256) w.bytes = 256;
  return w;
}

// Order key of a score: an unsigned integer that orders like the float
// (higher score -> larger key).  -0 and +0 are the same score (an IEEE tie,
// broken by the lower ID), so -0 is read as +0 before the bits are taken.
// NaN scores map to the key of -inf so that every round still picks a valid,
// untaken expert.  0 is below every key.
__device__ __forceinline__ uint32_t score_key(const float *l, const float *bias, int e) {
  float s = bias ? __fadd_rn(l[e], bias[e]) : l[e];
  if (s == 0.f) s = 0.f;
  if (isnan(s)) s = -INFINITY;
  const uint32_t b = __float_as_uint(s);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct RouteParams {
  const float *logits;
  const float *sel_bias;
  int64_t T;
  int E, k, renorm;
  uint32_t expert_start;
  int64_t chunk;
  float *weights;
  uint32_t *selected;
  int32_t *rank;      // [T*k] rank of (t, j) inside its chunk's rows of the same expert
  int32_t *hist;      // [nchunks][E]; single chunk: zeroed (the chunk base)
  int32_t *offsets;   // written when single != 0
  int single;
};

// R > 0: the E <= 32 R candidate keys of a lane stay in registers across the
// k selection rounds; R = 0 re-reads them each round (large E).
template <int R>
__global__ void __launch_bounds__(1024) route_rank_kernel(RouteParams p) {
  pdl_enter();  // programmatic dependent launch: the previous kernel is done
  extern __shared__ __align__(16) int32_t sm[];
  unsigned long long *mask = reinterpret_cast<unsigned long long *>(sm);  // [E] (64-token chunks)
  int32_t *cnt = reinterpret_cast<int32_t *>(mask + p.E);  // [E]
  int32_t *tmp = cnt + p.E;               // [32]
  int16_t *sel_s = reinterpret_cast<int16_t *>(tmp + 32);  // [chunk * k]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int64_t t0 = (int64_t)blockIdx.x * p.chunk;
  const int64_t t1 = min(p.T, t0 + p.chunk);
  const int E = p.E, k = p.k;
  for (int i = threadIdx.x; i < E; i += blockDim.x) {
    cnt[i] = 0;
    mask[i] = 0ull;
  }
  __syncthreads();

  for (int64_t t = t0 + warp; t < t1; t += nwarps) {
    const float *l = p.logits + t * E;
    // k rounds of (score desc, id asc) argmax over the candidates that come
    // after the previous winner in that order; two warp reductions a round
    uint32_t prev_key = 0xFFFFFFFFu;
    int prev_e = -1;
    int my_e = 0;  // lane j keeps the j-th selection
    if (R > 0) {
      // the lane's candidates (experts lane, lane + 32, ...) read once
      uint32_t keys[R > 0 ? R : 1];
#pragma unroll
      for (int i = 0; i < R; ++i) {
        const int e = lane + 32 * i;
        keys[i] = e < E ? score_key(l, p.sel_bias, e) : 0u;
      }
      for (int j = 0; j < k; ++j) {
        uint32_t bk = 0u;
        int be = 0x7FFFFFFF;
#pragma unroll
        for (int i = 0; i < R; ++i) {
          const int e = lane + 32 * i;
          const uint32_t key = keys[i];
          const bool after = key < prev_key || (key == prev_key && e > prev_e);
          if (e < E && after && key > bk) {  // ascending e per lane: a tie keeps the lower ID
            bk = key;
            be = e;
          }
        }
        const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
        const int we = (int)__reduce_min_sync(0xffffffffu, (bk == wk) ? (uint32_t)be : 0x7FFFFFFFu);
        prev_key = wk;
        prev_e = we;
        if (lane == j) my_e = we;
      }
    } else {
      for (int j = 0; j < k; ++j) {
        uint32_t bk = 0u;
        int be = 0x7FFFFFFF;
        for (int e = lane; e < E; e += 32) {
          const uint32_t key = score_key(l, p.sel_bias, e);
          const bool after = key < prev_key || (key == prev_key && e > prev_e);
          if (after && (key > bk || (key == bk && e < be))) {
            bk = key;
            be = e;
          }
        }
        const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
        const int we = (int)__reduce_min_sync(0xffffffffu, (bk == wk) ? (uint32_t)be : 0x7FFFFFFFu);
        prev_key = wk;
        prev_e = we;
        if (lane == j) my_e = we;
      }
    }
    // weights from the unbiased logits
    float lj = (lane < k) ? l[my_e] : -INFINITY;
    float m, den;
    if (p.renorm) {
      m = lj;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float ex = (lane < k) ? expf(lj - m) : 0.f;
      den = ex;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    } else {
      m = -INFINITY;
      for (int e = lane; e < E; e += 32) m = fmaxf(m, l[e]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      den = 0.f;
      for (int e = lane; e < E; e += 32) den += expf(l[e] - m);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    }
    if (lane < k) {
      p.weights[t * k + lane] = expf(lj - m) / den;
      p.selected[t * k + lane] = p.expert_start + (uint32_t)my_e;
      sel_s[(t - t0) * k + lane] = (int16_t)my_e;
      // a token picks an expert at most once: bit (t - t0) of the expert's mask
      if (p.chunk == 64) atomicOr(&mask[my_e], 1ull << (t - t0));
    }
  }
  __syncthreads();

  if (p.chunk == 64) {
    // rank of (t, j) among the chunk's rows of its expert = selecting tokens
    // before t (order-independent: the masks are complete)
    const int n = (int)(t1 - t0);
    for (int a = threadIdx.x; a < n * k; a += blockDim.x) {
      const int lt = a / k, e = sel_s[a];
      p.rank[(t0 + lt) * k + (a % k)] = __popcll(mask[e] & ((1ull << lt) - 1ull));
    }
    for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[i] = __popcll(mask[i]);
  } else if (warp == 0) {
    const int tpi = 32 / k;  // tokens per warp iteration
    const int n = (int)(t1 - t0);
    for (int tt = 0; tt < n; tt += tpi) {
      const int lt = tt + lane / k, j = lane % k;
      const bool active = lane < tpi * k && lt < n;
      const int e = active ? sel_s[lt * k + j] : -1 - lane;
      const unsigned grp = __match_any_sync(0xffffffffu, e);
      const int before = __popc(grp & ((1u << lane) - 1u));
      const int base = active ? cnt[e] : 0;
      __syncwarp();
      if (active) {
        p.rank[(t0 + lt) * k + j] = base + before;
        if ((grp >> lane) == 1u) cnt[e] = base + __popc(grp);  // highest lane of the group
      }
      __syncwarp();
    }
  }
  __syncthreads();

  if (!p.single) {
    for (int i = threadIdx.x; i < E; i += blockDim.x) p.hist[(int64_t)blockIdx.x * E + i] = cnt[i];
    return;
  }
  block_exclusive_scan(cnt, E, p.offsets, tmp);
  for (int i = threadIdx.x; i < E; i += blockDim.x) p.hist[i] = 0;
}

// Chunk bases (in place over hist) and offsets, one block.
__global__ void __launch_bounds__(kScanThreads) route_scan_kernel(int32_t *hist, int nch, int E,
                                                                   int32_t *offsets) {
  pdl_enter();  // programmatic dependent launch: the previous kernel is done
  extern __shared__ int32_t sm[];
  int32_t *totals = sm;                // [E]
  int32_t *tmp = totals + E;           // [32]
  int32_t *part = tmp + 32;            // [tpe * E] partial sums
  int tpe = 1;
  while (tpe * 2 * E <= (int)blockDim.x && tpe * 2 <= nch) tpe *= 2;
  const int cpp = (nch + tpe - 1) / tpe;  // chunks per part
  for (int u = threadIdx.x; u < tpe * E; u += blockDim.x) {
    int e = u % E, q = u / E;
    int c0 = q * cpp, c1 = min(nch, c0 + cpp);
    int32_t s = 0;
    for (int c = c0; c < c1; ++c) s += hist[(int64_t)c * E + e];
    part[q * E + e] = s;
  }
  __syncthreads();
  for (int u = threadIdx.x; u < tpe * E; u += blockDim.x) {
    int e = u % E, q = u / E;
    int32_t run = 0;
    for (int qq = 0; qq < q; ++qq) run += part[qq * E + e];
    if (q == tpe - 1) {
      int32_t tot = run + part[q * E + e];
      totals[e] = tot;
    }
    int c0 = q * cpp, c1 = min(nch, c0 + cpp);
    for (int c = c0; c < c1; ++c) {
      int32_t h = hist[(int64_t)c * E + e];
      hist[(int64_t)c * E + e] = run;
      run += h;
    }
  }
  __syncthreads();
  block_exclusive_scan(totals, E, offsets, tmp);
}

struct ScatterParams {
  const uint8_t *x;
  uint8_t *values;
  int64_t row_bytes;
  int64_t A;
  int k, E;
  uint32_t expert_start;
  int64_t chunk;
  const uint32_t *selected;
  const int32_t *offsets;
  const int32_t *chunk_base;
  const int32_t *rank;
  int32_t *row_of;
  uint32_t *row_experts;
  int32_t *src_token;
  int vec16;
  int64_t nseg;  // copy segments per row
  int32_t *status;
};

// Row position of assignment a = t*k + j and, on its first visit, the row maps.
__device__ __forceinline__ int64_t scatter_pos(const ScatterParams &p, int64_t a, bool write_maps) {
  const int64_t t = a / p.k;
  const int e = (int)(p.selected[a] - p.expert_start);
  const int64_t c = t / p.chunk;
  const int64_t pos = (int64_t)p.offsets[e] + p.chunk_base[c * p.E + e] + p.rank[a];
  if (write_maps) {
    p.row_of[a] = (int32_t)pos;
    p.row_experts[pos] = p.expert_start + (uint32_t)e;
    p.src_token[pos] = (int32_t)t;
  }
  return pos;
}

// 16-byte rows: one warp per assignment (grid-stride), four 512-byte
// segments loaded before they are stored.  Otherwise one warp per
// (assignment, 64-byte segment) with 2-byte accesses.  TO_F16: BF16 rows
// are written as F16 (exact in F16's normal range; a finite value above it
// or a NaN is reported as MOE_DEVICE_ERR_ACT_RANGE, as in the projections'
// own conversion).
template <bool TO_F16>
__global__ void __launch_bounds__(256) route_scatter_kernel(ScatterParams p) {
  pdl_enter();  // programmatic dependent launch: the previous kernel is done
  const int lane = threadIdx.x & 31;
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  if (!p.values) {  // row maps only (no COPY): one thread per assignment
    for (int64_t a = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; a < p.A; a += (int64_t)gridDim.x * blockDim.x)
      scatter_pos(p, a, true);
    return;
  }
  if (p.vec16) {
    const int64_t n16 = p.row_bytes / 16;
    for (int64_t a = wid; a < p.A; a += nw) {
      int64_t pos = 0;
      if (lane == 0) pos = scatter_pos(p, a, true);
      pos = __shfl_sync(0xffffffffu, pos, 0);
      const uint4 *src = reinterpret_cast<const uint4 *>(p.x + (a / p.k) * p.row_bytes);
      uint4 *dst = reinterpret_cast<uint4 *>(p.values + pos * p.row_bytes);
      uint32_t bad = 0;
      for (int64_t i0 = lane; i0 < n16; i0 += 32 * 4) {
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (i0 + 32 * j < n16) v[j] = __ldg(src + i0 + 32 * j);
        if (TO_F16) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (i0 + 32 * j < n16) act_quad_to_mt<__half>(v[j], MOE_BF16, bad);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (i0 + 32 * j < n16) dst[i0 + 32 * j] = v[j];
      }
      if (TO_F16 && bad) report(p.status, MOE_DEVICE_ERR_ACT_RANGE);
    }
    return;
  }
  const int64_t units = p.A * p.nseg;
  for (int64_t u = wid; u < units; u += nw) {
    const int64_t a = u / p.nseg, s = u % p.nseg;
    int64_t pos = 0;
    if (lane == 0) pos = scatter_pos(p, a, s == 0);
    pos = __shfl_sync(0xffffffffu, pos, 0);
    const uint8_t *src = p.x + (a / p.k) * p.row_bytes;
    uint8_t *dst = p.values + pos * p.row_bytes;
    const int64_t off = s * 64 + lane * 2;
    if (off < p.row_bytes) {
      uint16_t b = *reinterpret_cast<const uint16_t *>(src + off);
      if (TO_F16) {
        uint32_t bad = 0;
        b = (uint16_t)(act_pair_to_mt<__half>((uint32_t)b, MOE_BF16, bad) & 0xFFFFu);
        if (bad) report(p.status, MOE_DEVICE_ERR_ACT_RANGE);
      }
      *reinterpret_cast<uint16_t *>(dst + off) = b;
    }
  }
}

// Router-logit VJP at a fixed selection (one warp per token).
struct RouterBwdParams {
  const float *logits;
  const uint32_t *selected;
  const float *dw;
  int64_t T;
  int E, k, renorm;
  uint32_t expert_start;
  float *dl;
  int32_t *status;
};

__global__ void __launch_bounds__(256) router_bwd_kernel(RouterBwdParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= p.T) return;
  const float *l = p.logits + t * p.E;
  float *dl = p.dl + t * p.E;
  const int E = p.E, k = p.k;
  // lane j < k holds selection j
  int ej = -1;
  float lj = -INFINITY, dwj = 0.f;
  if (lane < k) {
    const uint32_t id = p.selected[t * k + lane];
    if (id >= p.expert_start && id - p.expert_start < (uint32_t)E) {
      ej = (int)(id - p.expert_start);
      lj = l[ej];
      dwj = p.dw[t * k + lane];
    } else {
      report(p.status, MOE_DEVICE_ERR_EXPERT_RANGE);
    }
  }
  float m, den;
  if (p.renorm) {
    m = lj;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    den = ej >= 0 ? expf(lj - m) : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  } else {
    m = -INFINITY;
    for (int e = lane; e < E; e += 32) m = fmaxf(m, l[e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    den = 0.f;
    for (int e = lane; e < E; e += 32) den += expf(l[e] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  }
  const float wj = ej >= 0 ? expf(lj - m) / den : 0.f;
  float dot = wj * dwj;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  if (p.renorm) {
    for (int e = lane; e < E; e += 32) dl[e] = 0.f;
    __syncwarp();
    if (ej >= 0) dl[ej] = wj * (dwj - dot);
  } else {
    for (int e = lane; e < E; e += 32) {
      float seed = 0.f;  // d_weights of the selection that chose e, if any
      for (int j = 0; j < k; ++j) {
        const int ejj = __shfl_sync(0xffffffffu, ej, j);
        const float dwjj = __shfl_sync(0xffffffffu, dwj, j);
        if (ejj == e) seed = dwjj;
      }
      dl[e] = expf(l[e] - m) / den * (seed - dot);
    }
  }
}

}  // namespace moe

using namespace moe;

// Host argument checks of moe_route_dispatch (and of its allocation-free
// variant, before its scratch-size check): MOE_OK or the error to return.
static moe_status route_check_args(const char *fn, const void *x, moe_dtype x_dtype, int64_t T, int64_t H,
                                   const float *logits, int64_t E, int32_t expert_start, int32_t top_k,
                                   const void *values, const float *weights, const uint32_t *selected_experts,
                                   const uint32_t *row_experts, const int32_t *offsets, const int32_t *src_token,
                                   const int32_t *row_of) {
  if (!valid_dtype(x_dtype)) return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "%s: bad x_dtype %d", fn, (int)x_dtype);
  if (T < 0 || H < 1 || E < 1 || E > MOE_MAX_EXPERTS)
    return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: bad sizes T=%lld H=%lld E=%lld", fn, (long long)T,
                     (long long)H, (long long)E);
  if (top_k < 1 || top_k > MOE_MAX_TOP_K || top_k > E)
    return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: top_k=%d outside [1, min(E, %d)]", fn, top_k, MOE_MAX_TOP_K);
  if (expert_start < 0 || (int64_t)expert_start + E > (int64_t)UINT32_MAX)
    return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: bad expert_start %d", fn, expert_start);
  if (!offsets) return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: offsets is NULL", fn);
  if (T == 0) return MOE_OK;
  if (!x || !logits || !values || !weights || !selected_experts || !row_experts || !src_token || !row_of)
    return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: NULL tensor pointer", fn);
  if (T * (int64_t)top_k > INT32_MAX)
    return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: T*top_k exceeds int32 row indices", fn);
  return MOE_OK;
}

extern "C" size_t moe_route_dispatch_workspace_size(int64_t T, int64_t E, int32_t top_k) {
  if (T < 0 || E < 1 || top_k < 1) return 0;
  return route_ws_layout(T, E, top_k).bytes;
}

// Routing, row maps and (values != NULL) the COPY of the rows; the two entry
// points below check their own arguments first.
static moe_status route_impl(const char *fn, const void *x, moe_dtype x_dtype, int64_t T, int64_t H,
                             const float *logits, const float *sel_bias, int64_t E, int32_t expert_start,
                             int32_t top_k, int32_t renormalize, void *values, bool to_f16, float *weights,
                             uint32_t *selected_experts, uint32_t *row_experts, int32_t *offsets,
                             int32_t *src_token, int32_t *row_of, void *workspace, size_t workspace_bytes,
                             int32_t *device_status, void *stream);

extern "C" moe_status moe_route_dispatch(const void *x, moe_dtype x_dtype, int64_t T, int64_t H,
                                         const float *logits, const float *sel_bias, int64_t E,
                                         int32_t expert_start, int32_t top_k, int32_t renormalize,
                                         void *values, float *weights, uint32_t *selected_experts,
                                         uint32_t *row_experts, int32_t *offsets, int32_t *src_token,
                                         int32_t *row_of, void *workspace, size_t workspace_bytes,
                                         int32_t *device_status, void *stream) {
  moe_status a = route_check_args("moe_route_dispatch", x, x_dtype, T, H, logits, E, expert_start, top_k, values,
                                  weights, selected_experts, row_experts, offsets, src_token, row_of);
  if (a != MOE_OK) return a;
  return route_impl("moe_route_dispatch", x, x_dtype, T, H, logits, sel_bias, E, expert_start, top_k, renormalize,
                    values, false, weights, selected_experts, row_experts, offsets, src_token, row_of, workspace,
                    workspace_bytes, device_status, stream);
}

extern "C" moe_status moe_route_dispatch_dt(const void *x, moe_dtype x_dtype, int64_t T, int64_t H,
                                            const float *logits, const float *sel_bias, int64_t E,
                                            int32_t expert_start, int32_t top_k, int32_t renormalize,
                                            void *values, moe_dtype values_dtype, float *weights,
                                            uint32_t *selected_experts, uint32_t *row_experts, int32_t *offsets,
                                            int32_t *src_token, int32_t *row_of, void *workspace,
                                            size_t workspace_bytes, int32_t *device_status, void *stream) {
  moe_status a = route_check_args("moe_route_dispatch", x, x_dtype, T, H, logits, E, expert_start, top_k, values,
                                  weights, selected_experts, row_experts, offsets, src_token, row_of);
  if (a != MOE_OK) return a;
  const bool to_f16 = x_dtype == MOE_BF16 && values_dtype == MOE_F16;
  if (values_dtype != x_dtype && !to_f16)
    return set_error(MOE_ERR_UNSUPPORTED_DTYPE, "moe_route_dispatch: values_dtype must be x_dtype, or F16 for BF16 x");
  return route_impl("moe_route_dispatch", x, x_dtype, T, H, logits, sel_bias, E, expert_start, top_k, renormalize,
                    values, to_f16, weights, selected_experts, row_experts, offsets, src_token, row_of, workspace,
                    workspace_bytes, device_status, stream);
}

extern "C" moe_status moe_route(const float *logits, const float *sel_bias, int64_t T, int64_t E,
                                int32_t expert_start, int32_t top_k, int32_t renormalize, float *weights,
                                uint32_t *selected_experts, uint32_t *row_experts, int32_t *offsets,
                                int32_t *src_token, int32_t *row_of, void *workspace, size_t workspace_bytes,
                                int32_t *device_status, void *stream) {
  (void)device_status;
  // the argument rules of moe_route_dispatch without x and values
  static const uint16_t kNoRows[8] = {};
  moe_status a = route_check_args("moe_route", kNoRows, MOE_BF16, T, 1, logits, E, expert_start, top_k, kNoRows,
                                  weights, selected_experts, row_experts, offsets, src_token, row_of);
  if (a != MOE_OK) return a;
  return route_impl("moe_route", nullptr, MOE_BF16, T, 1, logits, sel_bias, E, expert_start, top_k, renormalize,
                    nullptr, false, weights, selected_experts, row_experts, offsets, src_token, row_of, workspace,
                    workspace_bytes, nullptr, stream);
}

static moe_status route_impl(const char *fn, const void *x, moe_dtype x_dtype, int64_t T, int64_t H,
                             const float *logits, const float *sel_bias, int64_t E, int32_t expert_start,
                             int32_t top_k, int32_t renormalize, void *values, bool to_f16, float *weights,
                             uint32_t *selected_experts, uint32_t *row_experts, int32_t *offsets,
                             int32_t *src_token, int32_t *row_of, void *workspace, size_t workspace_bytes,
                             int32_t *device_status, void *stream) {
  cudaStream_t st = as_stream(stream);
  if (T == 0) {
    if (cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (size_t)(E + 1), st) != cudaSuccess)
      return check_launch("memset of the offsets");
    return MOE_OK;
  }
  RouteWs lay = route_ws_layout(T, E, top_k);
  if (!workspace || workspace_bytes < lay.bytes)
    return set_error(MOE_ERR_WORKSPACE, "%s: workspace of %zu bytes, need %zu", fn, workspace_bytes, lay.bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
    return set_error(MOE_ERR_INVALID_ARGUMENT, "%s: workspace not 16-byte aligned", fn);
  int32_t *hist = reinterpret_cast<int32_t *>(static_cast<char *>(workspace) + lay.hist_off);
  int32_t *rank = reinterpret_cast<int32_t *>(static_cast<char *>(workspace) + lay.rank_off);

  RouteParams rp;
  rp.logits = logits;
  rp.sel_bias = sel_bias;
  rp.T = T;
  rp.E = (int)E;
  rp.k = top_k;
  rp.renorm = renormalize ? 1 : 0;
  rp.expert_start = (uint32_t)expert_start;
  rp.chunk = lay.chunk;
  rp.weights = weights;
  rp.selected = selected_experts;
  rp.rank = rank;
  rp.hist = hist;
  rp.offsets = offsets;
  rp.single = lay.nchunks == 1;
  size_t smem = sizeof(unsigned long long) * (size_t)E + sizeof(int32_t) * (size_t)(E + 32) +
                sizeof(int16_t) * (size_t)(lay.chunk * top_k);
  smem = (smem + 15) & ~size_t(15);
  const int R = E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : E <= 256 ? 8 : E <= 512 ? 16 : 0;
  auto kern = R == 1 ? route_rank_kernel<1> : R == 2 ? route_rank_kernel<2> : R == 4 ? route_rank_kernel<4>
            : R == 8 ? route_rank_kernel<8> : R == 16 ? route_rank_kernel<16> : route_rank_kernel<0>;
  if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  // a warp per token (or per few tokens): the widest block the kernel takes
  const int threads = 1024;
  launch_pdl(kern, dim3((unsigned)lay.nchunks), dim3(threads), smem, st, rp);
  moe_status s = check_launch("route_rank_kernel");
  if (s != MOE_OK) return s;
  if (!rp.single) {
    int tpe = 1;
    while (tpe * 2 * E <= kScanThreads && tpe * 2 <= lay.nchunks) tpe *= 2;
    size_t ssm = sizeof(int32_t) * (size_t)(E + 32 + tpe * E);
    if (ssm > 48 * 1024) cudaFuncSetAttribute(route_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssm);
    launch_pdl(route_scan_kernel, dim3(1), dim3(kScanThreads), ssm, st, hist, (int)lay.nchunks, (int)E, offsets);
    s = check_launch("route_scan_kernel");
    if (s != MOE_OK) return s;
  }
  ScatterParams sp;
  sp.x = static_cast<const uint8_t *>(x);
  sp.values = static_cast<uint8_t *>(values);
  sp.row_bytes = H * dtype_bytes(x_dtype);
  sp.A = T * top_k;
  sp.k = top_k;
  sp.E = (int)E;
  sp.expert_start = (uint32_t)expert_start;
  sp.chunk = lay.chunk;
  sp.selected = selected_experts;
  sp.offsets = offsets;
  sp.chunk_base = hist;
  sp.rank = rank;
  sp.row_of = row_of;
  sp.row_experts = row_experts;
  sp.src_token = src_token;
  sp.vec16 = aligned16(x) && aligned16(values) && (sp.row_bytes % 16 == 0);
  sp.nseg = (sp.row_bytes + 63) / 64;  // 2-byte path only
  sp.status = device_status;
  int64_t units = !values ? (sp.A + 31) / 32 : sp.vec16 ? sp.A : sp.A * sp.nseg;
  int64_t blocks = (units + 7) / 8;
  int64_t cap = (int64_t)num_sms() * 16;
  if (blocks > cap) blocks = cap;
  if (to_f16)
    launch_pdl(route_scatter_kernel<true>, dim3((unsigned)blocks), dim3(256), 0, st, sp);
  else
    launch_pdl(route_scatter_kernel<false>, dim3((unsigned)blocks), dim3(256), 0, st, sp);
  return check_launch("route_scatter_kernel");
}

// ------------------------------------------------------------------ allocation-free variant
//
// Some callers cannot allocate device memory for a workspace: a serving
// loop that must not call cudaMalloc/cudaFree (they can synchronise the
// device and stall every stream), or a host framework that owns all device
// memory through its own pool and forbids allocations outside it.  For them
// the routing scratch lives in a fixed array compiled into this library.

#include <cudaTypedefs.h>

#include <mutex>

namespace moe {

constexpr size_t kStaticRouteScratchBytes = size_t(1) << 20;  // 1 MiB per device
static __device__ __align__(256) uint8_t g_route_scratch[kStaticRouteScratchBytes];

constexpr int kMaxScratchDevices = 64;
static std::mutex g_route_scratch_mu;
static void *g_route_scratch_ptr[kMaxScratchDevices] = {};
static unsigned long long g_route_scratch_ctx[kMaxScratchDevices] = {};

// Unique ID of the current CUDA context (0 if the driver cannot say).  A
// context made after cudaDeviceReset gets a new ID, and the library's device
// array a new address in it.
static unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_route_scratch on the current device.  Looked up once
// per device and context (the host-side name of the array is only a stand-in
// for the symbol); a new context on the device (after cudaDeviceReset) makes
// the next call look it up again.
static moe_status route_scratch_address(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxScratchDevices)
    return set_error(MOE_ERR_CUDA, "moe_route_dispatch_noalloc: no usable current device");
  // 0 before the runtime has made the device's context current: the lookup
  // below does that, and the ID is read again after it
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_route_scratch_mu);
  if (!g_route_scratch_ptr[dev] || ctx == 0 || ctx != g_route_scratch_ctx[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess || !p)
      return set_error(MOE_ERR_CUDA, "moe_route_dispatch_noalloc: cudaGetSymbolAddress failed: %s",
                       cudaGetErrorString(e));
    g_route_scratch_ptr[dev] = p;
    g_route_scratch_ctx[dev] = current_context_id();
  }
  *out = g_route_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace moe

extern "C" moe_status moe_route_dispatch_noalloc(const void *x, moe_dtype x_dtype, int64_t T, int64_t H,
                                                 const float *logits, const float *sel_bias, int64_t E,
                                                 int32_t expert_start, int32_t top_k, int32_t renormalize,
                                                 void *values, float *weights, uint32_t *selected_experts,
                                                 uint32_t *row_experts, int32_t *offsets, int32_t *src_token,
                                                 int32_t *row_of, int32_t *device_status, void *stream) {
  // the same argument errors as moe_route_dispatch, before the scratch check
  moe_status a = route_check_args("moe_route_dispatch_noalloc", x, x_dtype, T, H, logits, E, expert_start, top_k,
                                  values, weights, selected_experts, row_experts, offsets, src_token, row_of);
  if (a != MOE_OK) return a;
  const size_t need = route_ws_layout(T, E, top_k).bytes;
  if (need > kStaticRouteScratchBytes)
    return set_error(MOE_ERR_WORKSPACE,
                     "moe_route_dispatch_noalloc: T=%lld, E=%lld, top_k=%d need %zu bytes of scratch; the built-in "
                     "scratch holds %zu (use moe_route_dispatch with a workspace)",
                     (long long)T, (long long)E, top_k, need, kStaticRouteScratchBytes);
  void *scratch = nullptr;
  const moe_status s = route_scratch_address(&scratch);
  if (s != MOE_OK) return s;
  return moe_route_dispatch(x, x_dtype, T, H, logits, sel_bias, E, expert_start, top_k, renormalize, values,
                            weights, selected_experts, row_experts, offsets, src_token, row_of, scratch,
                            kStaticRouteScratchBytes, device_status, stream);
}

extern "C" moe_status moe_router_backward(const float *logits, const uint32_t *selected_experts,
                                          const float *d_weights, int64_t T, int64_t E, int32_t top_k,
                                          int32_t renormalize, int32_t expert_start, float *d_logits,
                                          int32_t *device_status, void *stream) {
  if (T < 0 || E < 1 || E > MOE_MAX_EXPERTS || top_k < 1 || top_k > MOE_MAX_TOP_K || top_k > E || expert_start < 0)
    return set_error(MOE_ERR_INVALID_ARGUMENT, "moe_router_backward: bad sizes T=%lld E=%lld top_k=%d",
                     (long long)T, (long long)E, top_k);
  if (T == 0) return MOE_OK;
  if (!logits || !selected_experts || !d_weights || !d_logits)
    return set_error(MOE_ERR_INVALID_ARGUMENT, "moe_router_backward: NULL tensor pointer");
  RouterBwdParams p{logits, selected_experts, d_weights, T, (int)E, top_k, renormalize ? 1 : 0,
                    (uint32_t)expert_start, d_logits, device_status};
  const int64_t blocks = (T * 32 + 255) / 256;
  router_bwd_kernel<<<(unsigned)blocks, 256, 0, as_stream(stream)>>>(p);
  return check_launch("moe_router_backward");
}
