// GELU through a table of Phi, shared by the activation kernel (quant.cu),
// the GEMM's requantising epilogue (gemm.cu) and the requantisation kernel.
// The table itself is the device array filled by quant.cu (ensure_gelu_table);
// kernels copy it into shared memory.
#pragma once

#include <cstdint>

namespace w4a4 {

// GELU table: Phi(t), the standard normal CDF, for the bf16 values t with
// exponent field kGeluFirstExp .. kGeluFirstExp + kGeluExps - 1
// (2^-12 <= |t| < 8), 128 mantissas each; entry 2 d + sign holds the value
// whose magnitude is the d-th of that range (the two signs side by side, so
// the sign bit lands in the byte offset with one shift and mask).
constexpr uint32_t kGeluFirstExp = 115;
constexpr uint32_t kGeluExps = 15;
constexpr int kGeluMags = static_cast<int>(kGeluExps * 128);   // magnitudes per sign
constexpr int kGeluTableSize = 2 * kGeluMags;

// GELU of the two bf16 inputs held in one 32-bit word: GELU(t) = t Phi(t)
// with Phi(t) = (1 + erf(t / sqrt 2)) / 2 read from the table (one product,
// so within about an ulp of the exact value).  The byte offsets of both
// entries are formed at once, one per 16-bit half (at most 8 * 1919 + 4, so
// no half overflows): the magnitude clamped with 16-bit SIMD min/max, minus
// the range start, times 8, plus 4 for a negative t; clamping the exponent field to the
// table's range is the only special case: below 2^-12 the entry of 2^-12
// stands in (Phi differs by < 1e-4, the product by < 3e-8 absolute), at or
// above 8 the entry of 8 - 2^-5 does, which holds 1 for positive t (Phi
// rounds to 1 there) and 0 for negative t, so GELU is t or -0 (the exact
// |t Phi(t)| is below 7e-15 for t <= -8 + 2^-5 and falls with |t|).  `tab`
// is the table in shared memory.
__device__ __forceinline__ void gelu_phi_word(uint32_t w, const float* __restrict__ tab, float& phi0, float& phi1) {
  constexpr uint32_t lo = kGeluFirstExp << 7, hi = ((kGeluFirstExp + kGeluExps) << 7) - 1u;
  uint32_t c;
  asm("max.u16x2 %0, %1, %2;" : "=r"(c) : "r"(w & 0x7FFF7FFFu), "r"(lo * 0x10001u));
  asm("min.u16x2 %0, %0, %1;" : "+r"(c) : "r"(hi * 0x10001u));
  const uint32_t off = ((c - lo * 0x10001u) << 3) | ((w >> 13) & 0x00040004u);
  const char* tb = reinterpret_cast<const char*>(tab);
  phi0 = *reinterpret_cast<const float*>(tb + (off & 0xFFFFu));
  phi1 = *reinterpret_cast<const float*>(tb + (off >> 16));
}


}  // namespace w4a4
