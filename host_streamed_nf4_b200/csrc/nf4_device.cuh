// nf4_device.cuh -- NF4 dequantization as the kernels do it.
//
// value(code) = bf16_rne(fp32(codebook[code] * absmax))   (one block = 64
// consecutive elements along k_in sharing one fp32 absmax; element e sits in
// byte e/2 of the code stream, even e in the high nibble).
//
// Instead of looking the codebook up per element, a thread builds the 16
// finished bf16 values of one block once (16 fp32 products, 8 paired
// round-to-nearest-even conversions) and splits them into a table of high
// bytes and a table of low bytes (4 registers each).  Each element is then a
// pure register permute (PRMT): no shared-memory traffic, which matters
// because the dequantizing warps share the SM's shared-memory bandwidth with
// the tensor cores reading their operands.  The product and the rounding are
// the same two IEEE operations for every element, so the result is the
// definition's, bit for bit.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace hsnf4 {

struct Nf4Codebook {
  float v[16];
};

struct Nf4Table {
  uint32_t h[4];  // h[i] byte j = high byte of the bf16 value of code 4i+j
  uint32_t l[4];  // l[i] byte j = low byte
};

__device__ __forceinline__ Nf4Table nf4_make_table(const Nf4Codebook& cb, float absmax) {
  uint32_t p[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    // low half = code 2j, high half = code 2j+1
    __nv_bfloat162 v = __floats2bfloat162_rn(__fmul_rn(cb.v[2 * j], absmax),
                                             __fmul_rn(cb.v[2 * j + 1], absmax));
    p[j] = *reinterpret_cast<uint32_t*>(&v);
  }
  Nf4Table t;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    t.h[i] = __byte_perm(p[2 * i], p[2 * i + 1], 0x7531);
    t.l[i] = __byte_perm(p[2 * i], p[2 * i + 1], 0x6420);
  }
  return t;
}

// Four codes held in the low 16 bits of x16 as they sit in memory (byte 0 =
// elements 0 (high nibble) and 1, byte 1 = elements 2 and 3) -> two words of
// bf16 pairs in element order: o0 = {e0, e1}, o1 = {e2, e3}.
__device__ __forceinline__ void nf4_lookup4(uint32_t x16, const Nf4Table& t, uint32_t& o0,
                                            uint32_t& o1) {
  // selector nibble j picks byte (code & 7) of an 8-entry half-table; bit 3 of
  // the code then picks the half.  PRMT reads bit 3 of a selector nibble as
  // "replicate sign", so it is cleared first.
  const uint32_t sel = x16 & 0x7777u;
  const uint32_t half = ((x16 >> 1) & 0x4444u) | 0x3210u;
  const uint32_t hlo = __byte_perm(t.h[0], t.h[1], sel);
  const uint32_t hhi = __byte_perm(t.h[2], t.h[3], sel);
  const uint32_t llo = __byte_perm(t.l[0], t.l[1], sel);
  const uint32_t lhi = __byte_perm(t.l[2], t.l[3], sel);
  const uint32_t hb = __byte_perm(hlo, hhi, half);  // byte j: nibble j's high byte
  const uint32_t lb = __byte_perm(llo, lhi, half);
  // nibbles 0..3 are elements 1, 0, 3, 2
  o0 = __byte_perm(lb, hb, 0x4051);
  o1 = __byte_perm(lb, hb, 0x6273);
}

// Eight codes (one little-endian word of the code stream) -> eight bf16.
__device__ __forceinline__ uint4 nf4_dequant8(uint32_t w, const Nf4Table& t) {
  uint4 r;
  nf4_lookup4(w & 0xFFFFu, t, r.x, r.y);
  nf4_lookup4(w >> 16, t, r.z, r.w);
  return r;
}

}  // namespace hsnf4
