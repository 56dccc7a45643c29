// BF16 -> F16 copy of an activation or gradient matrix, made once before a
// tcgen05 projection whose coefficients are F16 (the tensor-core operands
// of one MMA share a type).  Without it every column tile of the projection
// converts the same activation tile again in its dequant warps, which costs
// about as many instructions as forming the coefficients.  Exact in F16's
// normal range; a value F16 cannot hold (above its range, or NaN) is
// reported as MOE_DEVICE_ERR_ACT_RANGE, as the in-tile conversion does.
#include "proj.cuh"

namespace moe {

__global__ void __launch_bounds__(256) act_to_f16_kernel(const uint4 *src, uint4 *dst, int64_t n16,
                                                         int32_t *status) {
  pdl_enter();  // programmatic dependent launch: the previous kernel is done
  uint32_t bad = 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += stride) {
    uint4 v = __ldg(src + i);
    act_quad_to_mt<__half>(v, MOE_BF16, bad);
    dst[i] = v;
  }
  if (bad) report(status, MOE_DEVICE_ERR_ACT_RANGE);
}

// `elems` BF16 values (a multiple of 8, 16-byte aligned) from src into dst.
moe_status launch_act_to_f16(const void *src, void *dst, int64_t elems, int32_t *status, cudaStream_t st) {
  const int64_t n16 = elems / 8;
  if (n16 == 0) return MOE_OK;
  int64_t blocks = (n16 + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  launch_pdl(act_to_f16_kernel, dim3((unsigned)blocks), dim3(256), 0, st, static_cast<const uint4 *>(src),
             static_cast<uint4 *>(dst), n16, status);
  return check_launch("act_to_f16_kernel");
}

}  // namespace moe
