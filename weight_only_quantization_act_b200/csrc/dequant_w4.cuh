// dequant_w4.cuh - on-the-fly dequantization of packed 4-bit AWQ codes into a tensor-core operand tile
// ("GPU 硬件级反量化算子内联融合" on the bjdmk.com.cn AWQ article: unpack with shifts and masks, convert,
// apply the group's scale and offset). The value of code q in a group with step and zero point z is
// bf16(RN32(RN32(q - z) * step)), exactly the weight the quantizer's dequantization gives, rounded once
// to bf16 for the MMA.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace awq {

// Two fp32 lanes in one 64-bit register for the paired fp32 instructions of sm_100 (each lane is an
// ordinary IEEE operation rounded to nearest, so a pair gives exactly what two scalar operations give).
__device__ __forceinline__ uint64_t f32x2_pack(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ uint64_t f32x2_sub_mul(uint64_t a, uint64_t b, uint64_t c) {  // (a - b) * c
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;\n\tmul.rn.f32x2 %0, %0, %3;" : "=&l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(uint64_t v) {  // low lane -> low half, rounded to nearest
  uint32_t lo, hi, r;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "r"(hi), "r"(lo));
  return r;
}

// NW consecutive code words of one weight row (in-feature 8c+i at bits 4i..4i+3 of word c) -> 8 NW bf16
// values, packed two per register in in-feature order (o[4c + j] holds in-features 8c+2j, 8c+2j+1).
//
// Fast path (|z| < 2^19, every zero point a quantizer produces for sane weights): byte j of a word holds
// two codes; one byte permute puts the byte under the exponent bits of 2^23 (0x4B0000bb), and masking
// keeps the low nibble (the float 2^23 + q) or the high nibble in place (2^23 + 16 q). Subtracting
// 2^23 + z (resp. 2^23 + 16 z), both exact integers below 2^24, leaves q - z (resp. 16 (q - z)) exactly,
// and multiplying by step (resp. step / 16, an exact power-of-two scaling) rounds the same real product
// once. The two codes of a byte go through one paired subtract and one paired multiply. (Measured: the
// permute costs fewer ALU-pipe instructions per code than a shift per byte, and the ALU pipe is what
// bounds the dequantization.) Slow path (huge |z|): RN32(q - z) directly, as the quantizer defines it.
template <int NW>
__device__ __forceinline__ void dequant_words(const uint32_t (&w)[NW], float z, float stp, uint32_t (&o)[4 * NW]) {
  if (fabsf(z) < 524288.0f) {
    const float zb = __fadd_rn(8388608.0f, z);
    const float zb16 = __fadd_rn(8388608.0f, __fmul_rn(16.0f, z));
    const float st16 = __fmul_rn(stp, 0.0625f);
    const uint64_t zz = f32x2_pack(__float_as_uint(zb), __float_as_uint(zb16));
    const uint64_t ss = f32x2_pack(__float_as_uint(stp), __float_as_uint(st16));
#pragma unroll
    for (int c = 0; c < NW; ++c)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t t;  // 2^23 + byte j: byte j of the word under the exponent bits of 2^23
        asm("prmt.b32 %0, %1, %2, %3;" : "=r"(t) : "r"(w[c]), "r"(0x4B000000u), "r"(0x7650u | j));
        const uint64_t v = f32x2_pack(t & 0x4B00000Fu, t & 0x4B0000F0u);
        o[4 * c + j] = f32x2_to_bf16x2(f32x2_sub_mul(v, zz, ss));
      }
  } else {
#pragma unroll
    for (int c = 0; c < NW; ++c)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float q0 = static_cast<float>((w[c] >> (8 * j)) & 0xFu);
        const float q1 = static_cast<float>((w[c] >> (8 * j + 4)) & 0xFu);
        const __nv_bfloat162 pr =
            __floats2bfloat162_rn(__fmul_rn(__fsub_rn(q0, z), stp), __fmul_rn(__fsub_rn(q1, z), stp));
        o[4 * c + j] = *reinterpret_cast<const uint32_t*>(&pr);
      }
  }
}

// The values of dequant_words for words c0 .. c0+NW-1 of a row's k-block of 64 in-features, stored into
// the row's 128-byte line of a K-major tile with 128-byte swizzle: the 16-byte chunk of word c lands at
// chunk c ^ (row & 7) of the line at `line_addr`.
template <int NW>
__device__ __forceinline__ void store_words_sw128(const uint32_t (&o)[4 * NW], uint32_t line_addr, int row, int c0) {
  const uint32_t sw = static_cast<uint32_t>(row & 7);
#pragma unroll
  for (int c = 0; c < NW; ++c)
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(line_addr + ((static_cast<uint32_t>(c + c0) ^ sw) << 4)),
                 "r"(o[4 * c]), "r"(o[4 * c + 1]), "r"(o[4 * c + 2]), "r"(o[4 * c + 3])
                 : "memory");
}

}  // namespace awq
