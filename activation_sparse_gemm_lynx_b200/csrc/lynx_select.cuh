// lynx_select.cuh -- the 2:4 selection of a group of four bf16 values, shared
// by the sparsify pass and the fused GEMM.
//
// Per token row, each group of 4 consecutive values keeps its 2 largest
// magnitudes, ties to the lower position (RT-Lynx pages: qingkeai.online
// article, sections 02-03, Top-K 2:4 activation sparsity).  The selection of a
// group is decided by the six comparisons "x_i beats x_j" (i < j):
// |x_i| >= |x_j|, so a tie goes to the lower index.  They come out of three
// bf16x2 compares as a 6-bit code,
//   bit 0: |x0| >= |x2|   bit 1: |x0| >= |x3|   bit 2: |x0| >= |x1|
//   bit 3: |x1| >= |x3|   bit 4: |x1| >= |x2|   bit 5: |x2| >= |x3|,
// and a 64-entry table gives, per code, the byte selector that packs the two
// kept values (lower position in the low half) and the nibble lo | hi << 2.
// Value i is kept when fewer than two values beat it; a code that no order of
// four magnitudes produces maps to the two least beaten values.
#pragma once

#include <cstdint>

namespace lynx {

// acc_lo += low bf16 of w, acc_hi += high bf16 of w, in fp32 (one rounding
// each; the bf16 operand is exact in fp32)
__device__ __forceinline__ void add_bf16_pair(float& acc_lo, float& acc_hi, uint32_t w) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
      : "+f"(acc_lo), "+f"(acc_hi)
      : "r"(w));
}

// per 16-bit lane: 0xFFFF if a >= b, else 0 (bf16 compare; for the
// non-negative finite magnitudes used here the order of the bit patterns)
__device__ __forceinline__ uint32_t ge_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("set.ge.u32.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// The table entry of a selection code: the byte selector of the kept pair in
// bits 0-15, the nibble lo | hi << 2 in bits 16-19.
__device__ __forceinline__ uint32_t selection_table_entry(uint32_t code) {
  const int p02 = code & 1, p03 = (code >> 1) & 1, p01 = (code >> 2) & 1;
  const int p13 = (code >> 3) & 1, p12 = (code >> 4) & 1, p23 = (code >> 5) & 1;
  const int beaten[4] = {(1 - p01) + (1 - p02) + (1 - p03), p01 + (1 - p12) + (1 - p13),
                         p02 + p12 + (1 - p23), p03 + p13 + p23};
  int lo = -1, hi = -1;
  for (int limit = 0; limit <= 3 && hi < 0; ++limit)  // the least beaten first, lower index first
    for (int i = 0; i < 4 && hi < 0; ++i)
      if (beaten[i] == limit && i != lo) {
        if (lo < 0) lo = i;
        else hi = i;
      }
  if (hi < lo) {
    const int t = lo;
    lo = hi;
    hi = t;
  }
  const uint32_t sel = (2u * lo) | ((2u * lo + 1u) << 4) | ((2u * hi) << 8) | ((2u * hi + 1u) << 12);
  return sel | ((static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 2)) << 16);
}

// The selection code of the group with magnitude pairs a0 = |x1|:|x0| and
// a1 = |x3|:|x2| (sign bits cleared).
__device__ __forceinline__ uint32_t selection_code(uint32_t a0, uint32_t a1) {
  const uint32_t c1 = ge_bf16x2(a0, a1);                                // x0>=x2 | x1>=x3
  const uint32_t c2 = ge_bf16x2(a0, __byte_perm(a1, 0, 0x1032));        // x0>=x3 | x1>=x2
  const uint32_t c3 = ge_bf16x2(__byte_perm(a0, a1, 0x5410), __byte_perm(a0, a1, 0x7632));  // x0>=x1 | x2>=x3
  const uint32_t code = (c1 & 0x00010001u) | (c2 & 0x00020002u) | (c3 & 0x00040004u);
  return (code | (code >> 13)) & 0x3Fu;
}

// Top-2 of the group (w0 = x1:x0, w1 = x3:x2): returns the nibble lo | hi << 2
// and the kept pair packed (x_lo in the low half).
__device__ __forceinline__ uint32_t select_group_kept(uint32_t w0, uint32_t w1, const uint32_t* table,
                                                      uint32_t& kept) {
  const uint32_t ent = table[selection_code(w0 & 0x7FFF7FFFu, w1 & 0x7FFF7FFFu)];
  kept = __byte_perm(w0, w1, ent);
  return ent >> 16;
}

}  // namespace lynx
