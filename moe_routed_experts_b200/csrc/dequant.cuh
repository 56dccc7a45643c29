// Coefficient formation shared by the warp-tile kernels: AWQ words ->
// scale-dtype coefficient pairs in the register layouts the MMA fragments
// need (see the magic-number primitive in common.cuh).
#pragma once

#include "common.cuh"

namespace moe {

// Forward constants of one word column for one group: zero pairs
// (magic+z, magic+z) of logical columns 2p (zlo) and 2p+1 (zhi), and scale
// pairs (s, s) of the same columns.
template <typename MT>
struct FwdConsts {
  uint32_t zlo[4], zhi[4], slo[4], shi[4];
  __device__ __forceinline__ void load(uint32_t zw, uint4 sv) {
    constexpr uint32_t M = Dq<MT>::kMagic2;
    const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      // slots p (column 2p) and p+4 (column 2p+1) in the low/high halves
      const uint32_t t = (zw >> (4 * p)) & 0x000F000Fu;
      zlo[p] = prmt(t, 0u, 0x1010u) | M;  // (z[2p], z[2p]) under the magic
      zhi[p] = prmt(t, 0u, 0x3232u) | M;  // (z[2p+1], z[2p+1])
      slo[p] = prmt(sw[p], 0u, 0x1010u);  // (s[2p], s[2p])
      shi[p] = prmt(sw[p], 0u, 0x3232u);  // (s[2p+1], s[2p+1])
    }
  }
};

// The same constants with fewer instructions, for the streaming tile: the
// four zero-slot pairs come from shifts and masks, and each register is one
// byte permute of them under the magic number's high byte.
template <typename MT>
__device__ __forceinline__ void load_consts_fast(FwdConsts<MT> &c, uint32_t zw, uint4 sv) {
  constexpr uint32_t M = Dq<MT>::kMagic2;
  uint32_t t4[4];
  t4[0] = zw & 0x000F000Fu;
  t4[1] = (zw >> 4) & 0x000F000Fu;
  t4[2] = (zw >> 8) & 0x000F000Fu;
  t4[3] = (zw >> 12) & 0x000F000Fu;
  const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    // byte 0 (slot p) or byte 2 (slot p + 4) of t4[p], under the magic's high byte (byte 5 of {t4, M})
    c.zlo[p] = prmt(t4[p], M, 0x5050u);
    c.zhi[p] = prmt(t4[p], M, 0x5252u);
    c.slo[p] = prmt(sw[p], 0u, 0x1010u);
    c.shi[p] = prmt(sw[p], 0u, 0x3232u);
  }
}

// Coefficient pairs of column 2p (lo) and 2p+1 (hi) at two consecutive input
// rows, from the words wa (row kk) and wb (row kk+1) of the same column.
template <typename MT>
__device__ __forceinline__ void fwd_pairs(uint32_t wa, uint32_t wb, int p, const FwdConsts<MT> &c, uint32_t &lo,
                                          uint32_t &hi) {
  constexpr uint32_t M = Dq<MT>::kMagic2;
  const uint32_t u = prmt(wa, wb, 0x5410u);  // slots 0..3 of wa | slots 0..3 of wb
  const uint32_t v = prmt(wa, wb, 0x7632u);  // slots 4..7 of wa | slots 4..7 of wb
  lo = Dq<MT>::coef(nib_pair<M>(u >> (4 * p)), c.zlo[p], c.slo[p]);
  hi = Dq<MT>::coef(nib_pair<M>(v >> (4 * p)), c.zhi[p], c.shi[p]);
}

template <uint32_t kMask, uint32_t kMagic2>
__device__ __forceinline__ uint32_t nib_masked(uint32_t x) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "n"(kMask), "n"(kMagic2));
  return r;
}

// A fragments of one 16-row forward step, written out so that each permute
// and shift is formed once: a[q] = {col 2q rows (t, t+4), col 2q+1 rows
// (t, t+4), col 2q rows (t+8, t+12), col 2q+1 rows (t+8, t+12)} from the
// words w0..w3 of rows t, t+4, t+8, t+12.
template <typename MT>
__device__ __forceinline__ void fwd_step(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, const FwdConsts<MT> &c,
                                         uint32_t (&a)[4][4]) {
  constexpr uint32_t M = Dq<MT>::kMagic2;
  const uint32_t u01 = prmt(w0, w1, 0x5410u), v01 = prmt(w0, w1, 0x7632u);
  const uint32_t u23 = prmt(w2, w3, 0x5410u), v23 = prmt(w2, w3, 0x7632u);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    a[q][0] = Dq<MT>::coef(nib_masked<0x000F000Fu, M>(q ? u01 >> (4 * q) : u01), c.zlo[q], c.slo[q]);
    a[q][1] = Dq<MT>::coef(nib_masked<0x000F000Fu, M>(q ? v01 >> (4 * q) : v01), c.zhi[q], c.shi[q]);
    a[q][2] = Dq<MT>::coef(nib_masked<0x000F000Fu, M>(q ? u23 >> (4 * q) : u23), c.zlo[q], c.slo[q]);
    a[q][3] = Dq<MT>::coef(nib_masked<0x000F000Fu, M>(q ? v23 >> (4 * q) : v23), c.zhi[q], c.shi[q]);
  }
}

// Input-VJP extraction: coefficient pair of logical columns (2p, 2p+1) of one
// word, with zero word zw and the scale pair sp = (s[2p], s[2p+1]).
template <typename MT>
__device__ __forceinline__ uint32_t word_pair(uint32_t w, uint32_t zw, uint32_t sp, int p) {
  constexpr uint32_t M = Dq<MT>::kMagic2;
  return Dq<MT>::coef(nib_pair<M>(w >> (4 * p)), nib_pair<M>(zw >> (4 * p)), sp);
}

__device__ __forceinline__ uint4 ldg16(const uint16_t *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }

}  // namespace moe
