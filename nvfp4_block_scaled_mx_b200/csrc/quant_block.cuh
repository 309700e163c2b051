// quant_block.cuh -- the per-block quantization arithmetic shared by the streaming quantizer and
// the GEMM that quantizes its own activations (few-token linear layers): block amax on the bf16
// bit patterns, the MX scale exponent (EVEN / CEIL), the NVFP4 IEEE fp32 scale sequence, and the
// element encodes.
#pragma once

#include "mxq_device.cuh"

namespace mxq {

__device__ __forceinline__ uint32_t amax_bits16(const uint32_t* w, int n) {
    // max |bf16| over 2n values held as bf16x2 words, as an fp32 bit pattern
    uint32_t m = w[0] & 0x7FFF7FFFu;
    for (int i = 1; i < n; ++i) m = __vmaxu2(m, w[i] & 0x7FFF7FFFu);
    return max(m & 0xFFFFu, m >> 16) << 16;
}

// One NVFP4 block of 16 elements (8 bf16x2 words): the IEEE fp32 scale sequence t = fl(amax/6),
// u = fl(t/g), s = E4M3(u) (round to nearest even, saturating), d = fl(dec(s) * g), r = fl(1/d),
// then the elements fl(x * r) to E2M1.  d and r come from per-code tables (nvfp4_tables); s is at
// most 0x7E, as u is not negative and saturates to 448.  Writes 8 bytes of codes, returns s.
template <bool OBS>
__device__ __forceinline__ uint32_t nvfp4_block(const uint32_t* wb, float g, const float* tab_d, const float* tab_r,
                                                uint32_t* codes, uint32_t& seen) {
    const float amax = __uint_as_float(amax_bits16(wb, 8));
    if (OBS) seen = max(seen, __float_as_uint(amax));
    uint32_t s = 0;
    if (amax != 0.0f) {
        const float t = __fdiv_rn(amax, 6.0f);
        const float uu = __fdiv_rn(t, g);
        s = cvt_e4m3x2(uu, 0.0f) & 0xFFu;
    }
    const float r = tab_r[s];
    if (r == __int_as_float(0x7F800000)) {
        // r = fl(1/d) is +inf for d = 0 (every code a signed zero) and where 1/d overflows (d below
        // 2^-128, a subnormal g): x * r is then +-inf for x != 0, saturating to +-6, and a zero
        // element stays a signed zero
        const uint32_t big = tab_d[s] == 0.0f ? 0u : 7u;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t packed = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t v = wb[4 * h + i];
                packed |= ((v >> 15 & 1u) << 3 | ((v & 0x7FFFu) != 0 ? big : 0u)) << (8 * i);
                packed |= ((v >> 31) << 3 | ((v & 0x7FFF0000u) != 0 ? big : 0u)) << (8 * i + 4);
            }
            codes[h] = packed;
        }
    } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float f[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                f[2 * i] = __fmul_rn(__uint_as_float(wb[4 * h + i] << 16), r);
                f[2 * i + 1] = __fmul_rn(__uint_as_float(wb[4 * h + i] & 0xFFFF0000u), r);
            }
            codes[h] = cvt_e2m1x8(f);
        }
    }
    return s;
}

// d = fl(dec(s) * g) and r = fl(1/d) (+inf where d is 0) for the 128 non-negative E4M3 codes s,
// filled by the first 128 threads of a CTA.
__device__ __forceinline__ void nvfp4_tables(float g, float* tab_d, float* tab_r) {
    if (threadIdx.x < 128) {
        const float d = __fmul_rn(e4m3_decode_pos(threadIdx.x), g);
        tab_d[threadIdx.x] = d;
        tab_r[threadIdx.x] = __frcp_rn(d);  // correctly rounded 1/d, as fl(1/d); +inf for d = 0
    }
}

// Quantize one 32-element unit w (16 bf16x2 words): one MX block (MXFP4 / MXFP8) or two NVFP4
// blocks.  codes receives 4 words (FP4) or 8 words (FP8) of packed codes; the return value holds
// the scale byte (MX: the E8M0 code e + 127) or the two E4M3 scale bytes (NVFP4, first block low).
template <int FMT, int RULE, bool OBS>
__device__ __forceinline__ uint32_t quantize32(const uint32_t (&w)[16], float g, const float* tab_d, const float* tab_r,
                                               uint32_t* codes, uint32_t& seen) {
    if constexpr (FMT == MXQ_NVFP4) {
        const uint32_t s0 = nvfp4_block<OBS>(w, g, tab_d, tab_r, codes, seen);
        const uint32_t s1 = nvfp4_block<OBS>(w + 8, g, tab_d, tab_r, codes + 2, seen);
        return s0 | (s1 << 8);
    } else {
        constexpr int EMAX = (FMT == MXQ_MXFP8) ? 8 : 2;
        // CEIL moves one binade up when the amax mantissa exceeds elem_max's (1.5 for E2M1, 1.75 for E4M3)
        constexpr uint32_t MTHR = (FMT == MXQ_MXFP8) ? 0x600000u : 0x400000u;
        const uint32_t abits = amax_bits16(w, 16);
        int e = static_cast<int>(abits >> 23) - 127 - EMAX;
        if (RULE == MXQ_RULE_CEIL) e += ((abits & 0x7FFFFFu) > MTHR) ? 1 : 0;
        e = max(e, -127);
        const float inv = exp2_neg(e);
        if constexpr (FMT == MXQ_MXFP8) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float a0 = __fmul_rn(__uint_as_float(w[2 * i] << 16), inv);
                const float a1 = __fmul_rn(__uint_as_float(w[2 * i] & 0xFFFF0000u), inv);
                const float b0 = __fmul_rn(__uint_as_float(w[2 * i + 1] << 16), inv);
                const float b1 = __fmul_rn(__uint_as_float(w[2 * i + 1] & 0xFFFF0000u), inv);
                codes[i] = cvt_e4m3x2(a0, a1) | (cvt_e4m3x2(b0, b1) << 16);
            }
        } else {
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                float f[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    f[2 * i] = __fmul_rn(__uint_as_float(w[4 * h + i] << 16), inv);
                    f[2 * i + 1] = __fmul_rn(__uint_as_float(w[4 * h + i] & 0xFFFF0000u), inv);
                }
                codes[h] = cvt_e2m1x8(f);
            }
        }
        return static_cast<uint32_t>(e + 127);
    }
}

}  // namespace mxq
