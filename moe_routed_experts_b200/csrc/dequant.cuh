// Coefficient formation shared by the warp-tile kernels: AWQ words ->
// scale-dtype coefficient pairs in the register layouts the MMA fragments
// need (see the magic-number primitive in common.cuh).
#pragma once

#include "common.cuh"

namespace moe {

// Forward constants of one word column for one group: zero pairs
// (magic+z, magic+z) of logical columns 2p (zlo) and 2p+1 (zhi), and scale
// pairs (s, s) of the same columns.
//
// With x16 (F16 only, see fwd_pairs16) the zeros of the odd slots are taken
// 16 times larger, matching codes read in place from bits 4..7 of a byte.
template <typename MT>
struct FwdConsts {
  uint32_t zlo[4], zhi[4], slo[4], shi[4];
  __device__ __forceinline__ void load(uint32_t zw, uint4 sv, bool x16 = false) {
    constexpr uint32_t M = Dq<MT>::kMagic2;
    const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      // slots p (column 2p) and p+4 (column 2p+1) in the low/high halves
      uint32_t t = (zw >> (4 * p)) & 0x000F000Fu;
      if (x16 && (p & 1)) t <<= 4;
      zlo[p] = prmt(t, 0u, 0x1010u) | M;  // (z[2p], z[2p]) under the magic
      zhi[p] = prmt(t, 0u, 0x3232u) | M;  // (z[2p+1], z[2p+1])
      slo[p] = prmt(sw[p], 0u, 0x1010u);  // (s[2p], s[2p])
      shi[p] = prmt(sw[p], 0u, 0x3232u);  // (s[2p+1], s[2p+1])
    }
  }
};

// The same constants with fewer instructions, for the streaming tile: the
// four zero-slot pairs come from one shift and four masks (odd slots read in
// place when x16, 16 times larger, as the odd-slot codes are), and each
// register is one byte permute of them under the magic number's high byte.
template <typename MT>
__device__ __forceinline__ void load_consts_fast(FwdConsts<MT> &c, uint32_t zw, uint4 sv, bool x16) {
  constexpr uint32_t M = Dq<MT>::kMagic2;
  const uint32_t z8 = zw >> 8;
  uint32_t t4[4];
  t4[0] = zw & 0x000F000Fu;
  t4[1] = x16 ? (zw & 0x00F000F0u) : ((zw >> 4) & 0x000F000Fu);
  t4[2] = z8 & 0x000F000Fu;
  t4[3] = x16 ? (z8 & 0x00F000F0u) : ((zw >> 12) & 0x000F000Fu);
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

// Nonzero if a scale of the F16 pair is outside {0} U [2^-14, 256] (where the
// odd-slot shortcut of fwd_pairs16 would not be exact).
__device__ __forceinline__ uint32_t f16_pair_blocks_x16(uint32_t w) {
  const uint32_t lo = w & 0x7FFFu, hi = (w >> 16) & 0x7FFFu;
  return (uint32_t)(lo > 0x5C00u) | (uint32_t)(hi > 0x5C00u) | (uint32_t)(lo - 1u < 0x03FFu) |
         (uint32_t)(hi - 1u < 0x03FFu);
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

// F16 variant of fwd_pairs with fewer shifts: the code of an odd slot is
// used where it sits (bits 4..7 of its byte), so the lane holds 1024 + 16q
// (exact: below 2048) and the coefficient comes out as
// RNE(16 (q - z) s) = 16 RNE((q - z) s), exact whenever every nonzero
// product stays a normal F16 number before and after the scaling (the caller
// checks s = 0 or 2^-14 <= |s| <= 256; a subnormal product would be rounded
// on a coarser grid than its 16-times-larger normal image).  The MMAs of the odd
// slots therefore accumulate 16 times the true sum, which the caller
// rescales by 1/16 (exact) at the end.
__device__ __forceinline__ void fwd_pairs16(uint32_t wa, uint32_t wb, int p, const FwdConsts<__half> &c,
                                            uint32_t &lo, uint32_t &hi) {
  constexpr uint32_t M = Dq<__half>::kMagic2;
  const uint32_t u = prmt(wa, wb, 0x5410u), v = prmt(wa, wb, 0x7632u);
  const uint32_t us = (p >= 2) ? (u >> 8) : u, vs = (p >= 2) ? (v >> 8) : v;
  const uint32_t mask = (p & 1) ? 0x00F000F0u : 0x000F000Fu;
  uint32_t qu, qv;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(qu) : "r"(us), "r"(mask), "n"(M));
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(qv) : "r"(vs), "r"(mask), "n"(M));
  lo = Dq<__half>::coef(qu, c.zlo[p], c.slo[p]);
  hi = Dq<__half>::coef(qv, c.zhi[p], c.shi[p]);
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
// words w0..w3 of rows t, t+4, t+8, t+12.  X16 (F16 only): odd slots are
// read in place and come out 16 times larger (see fwd_pairs16).
template <typename MT, bool X16>
__device__ __forceinline__ void fwd_step(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, const FwdConsts<MT> &c,
                                         uint32_t (&a)[4][4]) {
  constexpr uint32_t M = Dq<MT>::kMagic2;
  const uint32_t u01 = prmt(w0, w1, 0x5410u), v01 = prmt(w0, w1, 0x7632u);
  const uint32_t u23 = prmt(w2, w3, 0x5410u), v23 = prmt(w2, w3, 0x7632u);
  uint32_t qu01[4], qv01[4], qu23[4], qv23[4];
  if (X16) {
    const uint32_t su01 = u01 >> 8, sv01 = v01 >> 8, su23 = u23 >> 8, sv23 = v23 >> 8;
    qu01[0] = nib_masked<0x000F000Fu, M>(u01);
    qu01[1] = nib_masked<0x00F000F0u, M>(u01);
    qu01[2] = nib_masked<0x000F000Fu, M>(su01);
    qu01[3] = nib_masked<0x00F000F0u, M>(su01);
    qv01[0] = nib_masked<0x000F000Fu, M>(v01);
    qv01[1] = nib_masked<0x00F000F0u, M>(v01);
    qv01[2] = nib_masked<0x000F000Fu, M>(sv01);
    qv01[3] = nib_masked<0x00F000F0u, M>(sv01);
    qu23[0] = nib_masked<0x000F000Fu, M>(u23);
    qu23[1] = nib_masked<0x00F000F0u, M>(u23);
    qu23[2] = nib_masked<0x000F000Fu, M>(su23);
    qu23[3] = nib_masked<0x00F000F0u, M>(su23);
    qv23[0] = nib_masked<0x000F000Fu, M>(v23);
    qv23[1] = nib_masked<0x00F000F0u, M>(v23);
    qv23[2] = nib_masked<0x000F000Fu, M>(sv23);
    qv23[3] = nib_masked<0x00F000F0u, M>(sv23);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      qu01[q] = nib_masked<0x000F000Fu, M>(q ? u01 >> (4 * q) : u01);
      qv01[q] = nib_masked<0x000F000Fu, M>(q ? v01 >> (4 * q) : v01);
      qu23[q] = nib_masked<0x000F000Fu, M>(q ? u23 >> (4 * q) : u23);
      qv23[q] = nib_masked<0x000F000Fu, M>(q ? v23 >> (4 * q) : v23);
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    a[q][0] = Dq<MT>::coef(qu01[q], c.zlo[q], c.slo[q]);
    a[q][1] = Dq<MT>::coef(qv01[q], c.zhi[q], c.shi[q]);
    a[q][2] = Dq<MT>::coef(qu23[q], c.zlo[q], c.slo[q]);
    a[q][3] = Dq<MT>::coef(qv23[q], c.zhi[q], c.shi[q]);
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
