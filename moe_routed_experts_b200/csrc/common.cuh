// Shared helpers of the CUDA library: host error reporting, storage-dtype
// loads and stores, device status flags, and the AWQ coefficient primitive
// used by every projection kernel.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "moe_awq.h"

namespace moe {

// ---------------------------------------------------------------- host side

moe_status set_error(moe_status s, const char *fmt, ...);
moe_status check_launch(const char *what);
inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int dtype_bytes(moe_dtype d) { return d == MOE_F32 ? 4 : 2; }
inline bool valid_dtype(int d) { return d == MOE_F32 || d == MOE_F16 || d == MOE_BF16; }
int num_sms();

// Launch with programmatic dependent launch: the kernel may be scheduled
// while the previous kernel of the stream is still finishing; its first
// statement (pdl_wait) then waits for that kernel's completion and memory,
// and pdl_trigger lets the next kernel be scheduled in turn.  Saves the
// launch gap and the tail of each kernel in the forward chain.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------- device side

// Wait for the previous kernel of the stream (its writes visible), then
// allow the next one to be scheduled.  No-ops without programmatic launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_enter() {
  pdl_wait();
  pdl_trigger();
}

__device__ __forceinline__ void report(int32_t *status, int bits) {
  if (status) atomicOr(status, bits);
}

__device__ __forceinline__ float ld_as_float(const void *base, int dt, int64_t i) {
  if (dt == MOE_F32) return reinterpret_cast<const float *>(base)[i];
  uint16_t b = reinterpret_cast<const uint16_t *>(base)[i];
  if (dt == MOE_BF16) return __uint_as_float(uint32_t(b) << 16);
  return __half2float(__ushort_as_half(b));
}

// Round-to-nearest-even FP32 -> storage dtype bits.
__device__ __forceinline__ uint16_t f32_to_bits(float v, int dt) {
  if (dt == MOE_BF16) return __bfloat16_as_ushort(__float2bfloat16_rn(v));
  return __half_as_ushort(__float2half_rn(v));
}

__device__ __forceinline__ float bits_to_f32(uint16_t b, int dt) {
  if (dt == MOE_BF16) return __uint_as_float(uint32_t(b) << 16);
  return __half2float(__ushort_as_half(b));
}

// ---------------------------------------------------------------- AWQ coefficients
//
// A pair register holds two 16-bit lanes.  `q` carries two 4-bit codes in
// bits 0..3 and 16..19.  OR-ing them under the bit pattern of a power of two
// whose binade has unit spacing (1024 for F16, 128 for BF16) gives the
// floats 1024+q (or 128+q) exactly; subtracting 1024+z (128+z) gives q-z
// exactly; multiplying by the scale rounds (q-z)*s once, in the scale dtype.
// This is the int->float "magic number" conversion (Kim et al., "Who Says
// Elephants Can't Run", 2022), used here only to form q-z exactly.

template <typename MT>
struct Dq;

template <>
struct Dq<__half> {
  static constexpr uint32_t kMagic2 = 0x64006400u;  // 1024.0 in both lanes
  __device__ __forceinline__ static uint32_t coef(uint32_t q_or_magic, uint32_t zc, uint32_t sc) {
    uint32_t d, c;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(q_or_magic), "r"(zc));
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(c) : "r"(d), "r"(sc));
    return c;
  }
};

template <>
struct Dq<__nv_bfloat16> {
  static constexpr uint32_t kMagic2 = 0x43004300u;  // 128.0 in both lanes
  __device__ __forceinline__ static uint32_t coef(uint32_t q_or_magic, uint32_t zc, uint32_t sc) {
    uint32_t d, c;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(q_or_magic), "r"(zc));
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(c) : "r"(d), "r"(sc));
    return c;
  }
};

// (x & 0x000F000F) | magic in one LOP3.
template <uint32_t kMagic2>
__device__ __forceinline__ uint32_t nib_pair(uint32_t x) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "n"(0x000F000Fu), "n"(kMagic2));
  return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Two BF16 (bits) -> two F16 (bits), through FP32; exact in F16's normal range.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  float lo = __uint_as_float(v << 16), hi = __uint_as_float(v & 0xFFFF0000u);
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}
// Two F16 -> two BF16 (rounds to BF16's 8 significant bits).
__device__ __forceinline__ uint32_t f16x2_to_bf16x2(uint32_t v) {
  __half2 h = *reinterpret_cast<__half2 *>(&v);
  float2 f = __half22float2(h);
  __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
  return *reinterpret_cast<uint32_t *>(&b);
}

// Activation (or gradient) pair in the tensor-core operand dtype MT.  A
// BF16 -> F16 conversion that changes a value grossly ORs 1 into `bad` (the
// caller reports MOE_DEVICE_ERR_ACT_RANGE): a finite value above F16's range
// (it becomes inf) or a NaN.  Values below F16's normal range keep what
// F16's subnormal grid holds (an absolute change below 2^-25, not reported);
// F16 -> BF16 always fits the range and rounds to BF16's 8 significant bits.
template <typename MT>
__device__ __forceinline__ uint32_t act_pair_to_mt(uint32_t v, int act_dt, uint32_t &bad) {
  if constexpr (sizeof(MT) == 2 && std::is_same<MT, __half>::value) {
    if (act_dt != MOE_BF16) return v;
    const uint32_t r = bf16x2_to_f16x2(v);
    // result inf/NaN in a lane whose source is not +-inf
    const uint32_t lo_bad = ((r & 0x7C00u) == 0x7C00u) & ((v & 0x7FFFu) != 0x7F80u);
    const uint32_t hi_bad = ((r & 0x7C000000u) == 0x7C000000u) & ((v & 0x7FFF0000u) != 0x7F800000u);
    bad |= lo_bad | hi_bad;
    return r;
  } else {
    return act_dt == MOE_F16 ? f16x2_to_bf16x2(v) : v;
  }
}

// Lane-wise maximum of two 16-bit pairs.
__device__ __forceinline__ uint32_t umax16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// N activation pairs at once, with the range report of act_pair_to_mt at a
// fraction of its cost: the pairs are tested one by one only when some
// source magnitude is at least 65536 (BF16 0x4780, the first value F16
// cannot hold; +-inf and NaN lie above it).  v << 1 doubles each 16-bit
// lane's magnitude (the low lane's sign moves into bit 0 of the high lane,
// which cannot carry it across the even threshold 0x8F00).
template <typename MT, int N>
__device__ __forceinline__ void act_pairs_to_mt(uint32_t (&v)[N], int act_dt, uint32_t &bad) {
  if constexpr (std::is_same<MT, __half>::value) {
    if (act_dt != MOE_BF16) return;
    uint32_t m = v[0] << 1;
#pragma unroll
    for (int i = 1; i < N; ++i) m = umax16x2(m, v[i] << 1);
    if ((umax16x2(m, m >> 16) & 0xFFFFu) >= 0x8F00u) {  // the larger lane
#pragma unroll
      for (int i = 0; i < N; ++i) v[i] = act_pair_to_mt<MT>(v[i], act_dt, bad);
      return;
    }
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = bf16x2_to_f16x2(v[i]);
  } else {
    if (act_dt != MOE_F16) return;
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = f16x2_to_bf16x2(v[i]);
  }
}

template <typename MT>
__device__ __forceinline__ void act_quad_to_mt(uint4 &q, int act_dt, uint32_t &bad) {
  uint32_t v[4] = {q.x, q.y, q.z, q.w};
  act_pairs_to_mt<MT, 4>(v, act_dt, bad);
  q = make_uint4(v[0], v[1], v[2], v[3]);
}

// mma.sync m16n8k16, FP32 accumulate.
template <typename MT>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (std::is_same<MT, __half>::value) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

__device__ __forceinline__ uint32_t ldg_nc_u32(const int32_t *p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.b32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// Block-wide exclusive scan of cnt[0..n) (in shared memory) into out[0..n],
// out[n] = total.  All threads of the block must call it.
__device__ __forceinline__ void block_exclusive_scan(const int32_t *cnt, int n, int32_t *out, int32_t *tmp) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int per = (n + nt - 1) / nt;
  const int b = tid * per, e = min(n, b + per);
  int32_t local = 0;
  for (int i = b; i < e; ++i) local += cnt[i];
  // warp inclusive scan
  const int lane = tid & 31, warp = tid >> 5;
  int32_t v = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int32_t u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) tmp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int nw = nt >> 5;
    int32_t w = lane < nw ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int32_t u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    if (lane < nw) tmp[lane] = w;
  }
  __syncthreads();
  int32_t run = v - local + (warp > 0 ? tmp[warp - 1] : 0);
  for (int i = b; i < e; ++i) {
    out[i] = run;
    run += cnt[i];
  }
  if (tid == nt - 1) out[n] = run;  // the last thread's range ends at n (or is empty)
  __syncthreads();
}

// Offsets check shared by the projection kernels: returns the row range of
// local expert e, or an empty range (and a status bit) if the mapping is
// inconsistent.
__device__ __forceinline__ bool expert_rows(const int32_t *offsets, int E, int64_t A, int e,
                                            int32_t *status, int64_t &r0, int64_t &r1) {
  int32_t a = offsets[e], b = offsets[e + 1];
  bool bad = (a < 0) || (b < a) || (int64_t)b > A || (e == 0 && a != 0) || (e == E - 1 && (int64_t)b != A);
  if (bad) {
    if (threadIdx.x == 0) report(status, MOE_DEVICE_ERR_OFFSETS);
    r0 = r1 = 0;
    return false;
  }
  r0 = a;
  r1 = b;
  return true;
}

}  // namespace moe
