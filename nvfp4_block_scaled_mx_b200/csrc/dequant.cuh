// dequant.cuh -- decoding packed FP4 / FP8 element codes back to bf16, shared by the W4A16 GEMM
// (weights dequantized into shared memory) and fake quantization (quantize, then decode).  Each
// routine turns one 32-bit word of codes into bf16x2 words, first element in the low half.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "mxq_device.cuh"

namespace mxq {

// 2^e as fp32 for e in [-127, 127] (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float pow2f(int e) {
    return e <= -127 ? __uint_as_float(0x00400000u) : __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
}

// 8 E2M1 codes (one 32-bit word, first element in the low nibble) times `scale`, as 4 bf16x2 words,
// through the conversion pipe (cvt e2m1x2 -> f16x2, fp32 multiply, cvt -> bf16x2).  Exact for every
// scale; used where the bf16 product could leave the normal range.
__device__ __forceinline__ uint4 dequant8_cvt(uint32_t w, float scale) {
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t h = e2m1x2_to_f16x2((w >> (8 * i)) & 0xFFu);
        const __half2 hh = *reinterpret_cast<const __half2*>(&h);
        const __nv_bfloat162 b =
            __floats2bfloat162_rn(__fmul_rn(__low2float(hh), scale), __fmul_rn(__high2float(hh), scale));
        o[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Byte permute: result byte i is byte sel_i of the 8-byte pair {b, a} (a is bytes 0-3).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// dequant8_cvt on the integer and FMA pipes.  Codes 2i and 2i+1 of the word are moved to bits 0-3 and
// 16-19 of one register (byte permute; selector nibbles 8-B yield zero bytes, as the selected bytes
// have a clear top bit), one integer multiply by 2^6 + 2^12 copies each code to bits 6-9 and 12-15
// (no carries: the copies do not overlap), and a mask keeps the magnitude bits at 6-8 and the sign
// at bit 15.  That bf16 pattern s<<15 | m<<6 reads as the code's value times 2^-126 (0.5 is the
// subnormal 0x0040), so a bf16x2 multiply by f2 = (2^126 s, 2^126 s) yields the scaled elements,
// exactly whenever every product is a normal bf16.
__device__ __forceinline__ uint4 dequant8_mul(uint32_t w, uint32_t f2) {
    const uint32_t ev = w & 0x0F0F0F0Fu;         // codes 0, 2, 4, 6 in the low nibbles of bytes 0-3
    const uint32_t od = (w >> 4) & 0x0F0F0F0Fu;  // codes 1, 3, 5, 7
    const uint32_t z[4] = {prmt(ev, od, 0x8480u), prmt(ev, od, 0x9591u), prmt(ev, od, 0xA6A2u), prmt(ev, od, 0xB7B3u)};
    const __nv_bfloat162 f = *reinterpret_cast<const __nv_bfloat162*>(&f2);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t t = (z[i] * 0x1040u) & 0x81C081C0u;
        const __nv_bfloat162 v = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&t), f);
        o[i] = *reinterpret_cast<const uint32_t*>(&v);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// f2 for an MXFP4 block with E8M0 code x: 2^126 * 2^(x - 127) = 2^(x - 1), a normal bf16 for x in
// [1, 128]; every product is then normal and exact for x in [2, 128].
__device__ __forceinline__ uint32_t mx_factor2(uint32_t x) { return ((x + 126u) << 7) * 0x10001u; }


// bf16x2 (2^126, 2^126): dequant8_mul by this factor yields the E2M1 element values themselves.
constexpr uint32_t kE2m1Unit2 = 0x7E807E80u;

// 8 E2M1 codes times an arbitrary fp32 d, rounded as fl32(elem * d) and then to bf16 (RNE): the
// elements come out of dequant8_mul exactly, are widened to fp32 (a bf16 is the high half of its
// fp32), multiplied and packed.  Exact in the same sense as dequant8_cvt, on the FMA pipe.
__device__ __forceinline__ uint4 dequant8_fmul(uint32_t w, float d) {
    const uint4 e = dequant8_mul(w, kE2m1Unit2);
    const uint32_t ew[4] = {e.x, e.y, e.z, e.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(ew[i] << 16), d),
                                                       __fmul_rn(__uint_as_float(ew[i] & 0xFFFF0000u), d));
        o[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// 4 E4M3 codes (one word, first element in the low byte) times the bf16x2 factor f2, as 2 bf16x2
// words.  Each code byte is moved to the high byte of a 16-bit half (byte permute), and its seven
// magnitude bits are shifted down by 4 under the sign: the bf16 pattern s<<15 | (eeee mmm)<<4 reads
// as the code's value times 2^-120 (E4M3 subnormals land on bf16 subnormals, the same scaling), so
// with f2 = 2^120 s the products are the scaled elements, exact whenever each is a normal bf16.
__device__ __forceinline__ uint2 e4m3x4_mul(uint32_t c, uint32_t f2) {
    const uint32_t z[2] = {prmt(c, 0u, 0x1404u), prmt(c, 0u, 0x3424u)};
    const __nv_bfloat162 f = *reinterpret_cast<const __nv_bfloat162*>(&f2);
    uint32_t o[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint32_t t = (z[i] & 0x80008000u) | ((z[i] >> 4) & 0x07F007F0u);
        const __nv_bfloat162 v = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&t), f);
        o[i] = *reinterpret_cast<const uint32_t*>(&v);
    }
    return make_uint2(o[0], o[1]);
}

// f2 for an MXFP8 block with E8M0 code x: 2^120 * 2^(x - 127) = 2^(x - 7), a normal bf16 for x in
// [1, 134]; every product (|elem| >= 2^-9) is then normal and exact for x in [10, 134].
__device__ __forceinline__ uint32_t mx8_factor2(uint32_t x) { return ((x + 120u) << 7) * 0x10001u; }

}  // namespace mxq
