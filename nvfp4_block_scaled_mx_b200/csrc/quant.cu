// quant.cu -- bf16 -> MXFP4 (EVEN / CEIL), NVFP4 and MXFP8 block quantizer, scale swizzle,
// NVFP4 global scale, and the bounded-wait self-test kernel.
//
// The quantizer is a single streaming pass over x: each thread owns 32 consecutive elements of a
// row (four 16-byte loads; one MX block or two NVFP4 blocks), takes the block amax on the bf16 bit
// patterns, derives the scale, and writes 16 (FP4) or 32 (FP8) bytes of packed codes plus one scale
// byte per block, either row-major or directly in the swizzled tensor-core layout.
#include "mxq_device.cuh"
#include "mxq_internal.h"

namespace mxq {
namespace {

constexpr int kQuantThreads = 256;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Scale byte offset of block (row, kc) in the swizzled layout.
__device__ __forceinline__ uint32_t swz_offset(uint32_t row, uint32_t kc, uint32_t col_tiles) {
    return ((row >> 7) * col_tiles + (kc >> 2)) * 512u + (row & 31u) * 16u + ((row >> 5) & 3u) * 4u + (kc & 3u);
}

// floor(n / d) for n, d < 2^32 with magic = ceil(2^64 / d) (d > 1): the product's high word is
// exact because the rounding of the magic adds less than 2^-32 to n / d.
__device__ __forceinline__ uint32_t div_magic(uint32_t n, uint32_t d, uint64_t magic) {
    return d == 1 ? n : static_cast<uint32_t>(__umul64hi(static_cast<uint64_t>(n), magic));
}

// ld.global.nc with L1 allocation: the four 16-byte loads of a thread cover 64 contiguous bytes,
// so the sector halves one load leaves in L1 serve the next.
__device__ __forceinline__ uint4 ld_nc(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t amax_bits16(const uint32_t* w, int n) {
    // max |bf16| over 2n values held as bf16x2 words, as an fp32 bit pattern
    uint32_t m = w[0] & 0x7FFF7FFFu;
    for (int i = 1; i < n; ++i) m = __vmaxu2(m, w[i] & 0x7FFF7FFFu);
    return max(m & 0xFFFFu, m >> 16) << 16;
}

// Scale byte offset of block `blk` (row-major block index) in the requested layout.
template <bool SWZ>
__device__ __forceinline__ uint32_t scale_offset(uint32_t blk, uint32_t kblocks, uint64_t kb_magic, uint32_t col_tiles) {
    if constexpr (!SWZ) return blk;
    const uint32_t row = div_magic(blk, kblocks, kb_magic);
    const uint32_t kc = blk - row * kblocks;
    return swz_offset(row, kc, col_tiles);
}

// One thread quantizes 32 consecutive elements of a row: one MX block (MXFP4 / MXFP8) or two
// NVFP4 blocks.  Codes: 16 bytes (FP4) or 32 bytes (FP8) per thread, coalesced across the warp.
// OBS (NVFP4 only): gptr is a running amax; g = fl(amax / (6*448)) and the tensor amax of x is
// folded into *amax_out with one atomicMax per warp.
template <int FMT, int RULE, bool SWZ, bool OBS = false>
__global__ void __launch_bounds__(kQuantThreads, 8) quantize_kernel(const uint4* __restrict__ x, int64_t n_units,
                                                                 uint32_t kblocks, uint64_t kb_magic,
                                                                 uint32_t col_tiles,
                                                                 const float* __restrict__ gptr,
                                                                 uint8_t* __restrict__ q, uint8_t* __restrict__ sf,
                                                                 unsigned int* __restrict__ amax_out = nullptr) {
    pdl_launch_dependents();
    const float g = (FMT == MXQ_NVFP4) ? (OBS ? __fdiv_rn(*gptr, 2688.0f) : *gptr) : 1.0f;
    uint32_t seen = 0;  // largest block amax (fp32 bits) this thread quantized, for OBS
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < n_units; u += stride) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = ld_nc(x + u * 4 + i);
            w[4 * i + 0] = v.x;
            w[4 * i + 1] = v.y;
            w[4 * i + 2] = v.z;
            w[4 * i + 3] = v.w;
        }
        if constexpr (FMT == MXQ_NVFP4) {
            uint32_t codes[4];
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const uint32_t* wb = w + 8 * b;
                const float amax = __uint_as_float(amax_bits16(wb, 8));
                if (OBS) seen = max(seen, __float_as_uint(amax));
                uint32_t s = 0;
                if (amax != 0.0f) {
                    const float t = __fdiv_rn(amax, 6.0f);
                    const float uu = __fdiv_rn(t, g);
                    s = cvt_e4m3x2(uu, 0.0f) & 0xFFu;
                }
                const float d = __fmul_rn(e4m3_decode_pos(s), g);
                if (d == 0.0f) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t packed = 0;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            packed |= (wb[4 * h + i] >> 15 & 1u) << (8 * i + 3);
                            packed |= (wb[4 * h + i] >> 31) << (8 * i + 7);
                        }
                        codes[2 * b + h] = packed;
                    }
                } else {
                    const float r = __frcp_rn(d);  // correctly rounded 1/d, as fl(1/d)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float f[8];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            f[2 * i] = __fmul_rn(__uint_as_float(wb[4 * h + i] << 16), r);
                            f[2 * i + 1] = __fmul_rn(__uint_as_float(wb[4 * h + i] & 0xFFFF0000u), r);
                        }
                        codes[2 * b + h] = cvt_e2m1x8(f);
                    }
                }
                sf[scale_offset<SWZ>(static_cast<uint32_t>(2 * u + b), kblocks, kb_magic, col_tiles)] =
                    static_cast<uint8_t>(s);
            }
            reinterpret_cast<uint4*>(q)[u] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
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
                uint32_t codes[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float a0 = __fmul_rn(__uint_as_float(w[2 * i] << 16), inv);
                    const float a1 = __fmul_rn(__uint_as_float(w[2 * i] & 0xFFFF0000u), inv);
                    const float b0 = __fmul_rn(__uint_as_float(w[2 * i + 1] << 16), inv);
                    const float b1 = __fmul_rn(__uint_as_float(w[2 * i + 1] & 0xFFFF0000u), inv);
                    codes[i] = cvt_e4m3x2(a0, a1) | (cvt_e4m3x2(b0, b1) << 16);
                }
                uint4* dst = reinterpret_cast<uint4*>(q) + 2 * u;
                dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
                dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
            } else {
                uint32_t codes[4];
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
                reinterpret_cast<uint4*>(q)[u] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
            }
            sf[scale_offset<SWZ>(static_cast<uint32_t>(u), kblocks, kb_magic, col_tiles)] = static_cast<uint8_t>(e + 127);
        }
    }
    if constexpr (OBS) {
        seen = __reduce_max_sync(0xFFFFFFFFu, seen);
        if ((threadIdx.x & 31) == 0 && seen != 0) atomicMax(amax_out, seen);
    }
}

template <int FMT, int RULE, bool SWZ>
cudaError_t launch_q(const void* x, int64_t M, int64_t K, const float* g, void* q, void* sf, cudaStream_t stream) {
    const int64_t n_units = M * K / 32;
    const uint32_t kblocks = static_cast<uint32_t>(K / block_size(FMT));
    const uint32_t col_tiles = static_cast<uint32_t>(ceil_div(kblocks, 4));
    int64_t blocks = ceil_div(n_units, static_cast<int64_t>(kQuantThreads));
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    // ceil(2^64 / kblocks); unused when kblocks == 1
    const uint64_t kb_magic =
        kblocks > 1 ? static_cast<uint64_t>(((static_cast<unsigned __int128>(1) << 64) + kblocks - 1) / kblocks) : 0;
    quantize_kernel<FMT, RULE, SWZ><<<static_cast<unsigned>(blocks), kQuantThreads, 0, stream>>>(
        static_cast<const uint4*>(x), n_units, kblocks, kb_magic, col_tiles, g, static_cast<uint8_t*>(q),
        static_cast<uint8_t*>(sf));
    return cudaGetLastError();
}

// ------------------------------------------------------------------ fake quantization

__device__ __forceinline__ float e2m1_decode(uint32_t c) {
    const uint32_t e = (c >> 1) & 3u, m = c & 1u;
    const float mag = e == 0 ? (m ? 0.5f : 0.0f) : __uint_as_float(((e + 126u) << 23) | (m << 22));
    return (c & 8u) ? -mag : mag;
}

__device__ __forceinline__ float e4m3_decode(uint32_t c) {
    const float mag = e4m3_decode_pos(c & 0x7Fu);
    return (c & 0x80u) ? -mag : mag;
}

// 2^e as fp32 for e in [-127, 126] (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float exp2_pos(int e) {
    return e <= -127 ? __uint_as_float(0x00400000u) : __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&b);
}

// One thread fake-quantizes 32 consecutive elements: the same codes and scales as quantize_kernel,
// decoded in the format's precision (MX: elem * 2^e, NVFP4: fl(elem * d)) and rounded once to bf16.
template <int FMT, int RULE>
__global__ void __launch_bounds__(kQuantThreads) fake_quantize_kernel(const uint4* x, int64_t n_units,
                                                                         const float* __restrict__ gptr, uint4* y) {
    const float g = (FMT == MXQ_NVFP4) ? *gptr : 1.0f;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < n_units; u += stride) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = ld_nc(x + u * 4 + i);
            w[4 * i + 0] = v.x;
            w[4 * i + 1] = v.y;
            w[4 * i + 2] = v.z;
            w[4 * i + 3] = v.w;
        }
        if constexpr (FMT == MXQ_NVFP4) {
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const uint32_t* wb = w + 8 * b;
                const float amax = __uint_as_float(amax_bits16(wb, 8));
                uint32_t s = 0;
                if (amax != 0.0f) s = cvt_e4m3x2(__fdiv_rn(__fdiv_rn(amax, 6.0f), g), 0.0f) & 0xFFu;
                const float d = __fmul_rn(e4m3_decode_pos(s), g);
                const float r = d == 0.0f ? 0.0f : __frcp_rn(d);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t codes;
                    if (d == 0.0f) {
                        codes = 0;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            codes |= (wb[4 * h + i] >> 15 & 1u) << (8 * i + 3);
                            codes |= (wb[4 * h + i] >> 31) << (8 * i + 7);
                        }
                    } else {
                        float f[8];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            f[2 * i] = __fmul_rn(__uint_as_float(wb[4 * h + i] << 16), r);
                            f[2 * i + 1] = __fmul_rn(__uint_as_float(wb[4 * h + i] & 0xFFFF0000u), r);
                        }
                        codes = cvt_e2m1x8(f);
                    }
                    uint32_t o[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        o[i] = pack_bf16x2(__fmul_rn(e2m1_decode(codes >> (8 * i)), d),
                                           __fmul_rn(e2m1_decode(codes >> (8 * i + 4)), d));
                    y[u * 4 + 2 * b + h] = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
        } else {
            constexpr int EMAX = (FMT == MXQ_MXFP8) ? 8 : 2;
            constexpr uint32_t MTHR = (FMT == MXQ_MXFP8) ? 0x600000u : 0x400000u;
            const uint32_t abits = amax_bits16(w, 16);
            int e = static_cast<int>(abits >> 23) - 127 - EMAX;
            if (RULE == MXQ_RULE_CEIL) e += ((abits & 0x7FFFFFu) > MTHR) ? 1 : 0;
            e = max(e, -127);
            const float inv = exp2_neg(e), sc = exp2_pos(e);
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float lo = __fmul_rn(__uint_as_float(w[i] << 16), inv);
                const float hi = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), inv);
                uint32_t& oi = o[i & 3];
                float dlo, dhi;
                if constexpr (FMT == MXQ_MXFP8) {
                    const uint32_t c = cvt_e4m3x2(lo, hi);
                    dlo = e4m3_decode(c & 0xFFu);
                    dhi = e4m3_decode(c >> 8);
                } else {
                    uint16_t c8;
                    asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %2, %1;\n\tcvt.u16.u8 %0, b;\n\t}\n"
                        : "=h"(c8)
                        : "f"(lo), "f"(hi));
                    dlo = e2m1_decode(c8 & 0xFu);
                    dhi = e2m1_decode(c8 >> 4);
                }
                oi = pack_bf16x2(__fmul_rn(dlo, sc), __fmul_rn(dhi, sc));
                if ((i & 3) == 3) y[u * 4 + (i >> 2)] = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
    }
}

template <int FMT, int RULE>
cudaError_t launch_fq(const void* x, int64_t M, int64_t K, const float* g, void* y, cudaStream_t stream) {
    const int64_t n_units = M * K / 32;
    int64_t blocks = ceil_div(n_units, static_cast<int64_t>(kQuantThreads));
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    fake_quantize_kernel<FMT, RULE><<<static_cast<unsigned>(blocks), kQuantThreads, 0, stream>>>(
        static_cast<const uint4*>(x), n_units, g, static_cast<uint4*>(y));
    return cudaGetLastError();
}

template <bool SWZ>
cudaError_t launch_q_running(const void* x, int64_t M, int64_t K, const float* amax_in, float* amax_out, void* q,
                             void* sf, cudaStream_t stream) {
    const int64_t n_units = M * K / 32;
    const uint32_t kblocks = static_cast<uint32_t>(K / 16);
    const uint32_t col_tiles = static_cast<uint32_t>(ceil_div(kblocks, 4));
    int64_t blocks = ceil_div(n_units, static_cast<int64_t>(kQuantThreads));
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    const uint64_t kb_magic =
        kblocks > 1 ? static_cast<uint64_t>(((static_cast<unsigned __int128>(1) << 64) + kblocks - 1) / kblocks) : 0;
    quantize_kernel<MXQ_NVFP4, 0, SWZ, true><<<static_cast<unsigned>(blocks), kQuantThreads, 0, stream>>>(
        static_cast<const uint4*>(x), n_units, kblocks, kb_magic, col_tiles, amax_in, static_cast<uint8_t*>(q),
        static_cast<uint8_t*>(sf), reinterpret_cast<unsigned int*>(amax_out));
    return cudaGetLastError();
}

template <bool SWZ>
cudaError_t launch_q_layout(const void* x, int64_t M, int64_t K, int fmt, int rule, const float* g, void* q, void* sf,
                            cudaStream_t stream) {
    if (fmt == MXQ_NVFP4) return launch_q<MXQ_NVFP4, 0, SWZ>(x, M, K, g, q, sf, stream);
    if (fmt == MXQ_MXFP8) {
        return rule == MXQ_RULE_CEIL ? launch_q<MXQ_MXFP8, MXQ_RULE_CEIL, SWZ>(x, M, K, g, q, sf, stream)
                                     : launch_q<MXQ_MXFP8, MXQ_RULE_EVEN, SWZ>(x, M, K, g, q, sf, stream);
    }
    return rule == MXQ_RULE_CEIL ? launch_q<MXQ_MXFP4, MXQ_RULE_CEIL, SWZ>(x, M, K, g, q, sf, stream)
                                 : launch_q<MXQ_MXFP4, MXQ_RULE_EVEN, SWZ>(x, M, K, g, q, sf, stream);
}

// ------------------------------------------------------------------ swizzle

__global__ void swizzle_kernel(const uint8_t* __restrict__ src, uint32_t rows, uint32_t kblocks, uint32_t col_tiles,
                               uint8_t* __restrict__ dst, int64_t total) {
    for (int64_t off = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; off < total;
         off += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const uint32_t tile = static_cast<uint32_t>(off >> 9), within = static_cast<uint32_t>(off & 511);
        const uint32_t rt = tile / col_tiles, ct = tile - rt * col_tiles;
        const uint32_t r = rt * 128u + ((within & 15u) >> 2) * 32u + (within >> 4);
        const uint32_t c = ct * 4u + (within & 3u);
        dst[off] = (r < rows && c < kblocks) ? src[static_cast<int64_t>(r) * kblocks + c] : 0;
    }
}

// ------------------------------------------------------------------ global scale

__global__ void amax_kernel(const uint4* __restrict__ x, int64_t n_chunks, const uint16_t* __restrict__ tail,
                            int n_tail, unsigned int* __restrict__ amax_bits) {
    uint32_t m = 0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_chunks;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const uint4 v = ld_stream(x + i);
        const uint32_t m2 = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                     __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
        m = max(m, max(m2 & 0xFFFFu, m2 >> 16));
    }
    if (blockIdx.x == 0 && static_cast<int>(threadIdx.x) < n_tail) m = max(m, static_cast<uint32_t>(tail[threadIdx.x] & 0x7FFFu));
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if ((threadIdx.x & 31) == 0 && m != 0) atomicMax(amax_bits, m << 16);
}

__global__ void global_scale_finalize(const float* amax, float* g) { *g = __fdiv_rn(*amax, 2688.0f); }

// ------------------------------------------------------------------ bounded-wait self-test

__global__ void selftest_timeout_kernel(int* status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    // phase 0 of this barrier never completes: nothing arrives on it
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, status, 99, limit_ns);
}

}  // namespace

cudaError_t launch_quantize(const void* x, int64_t M, int64_t K, int fmt, int rule, const float* g, void* q, void* sf,
                            int layout, cudaStream_t stream) {
    if (layout == MXQ_SF_SWIZZLED) {
        const int64_t kb = K / block_size(fmt);
        if (M % 128 != 0 || kb % 4 != 0) {
            cudaError_t e = cudaMemsetAsync(sf, 0, static_cast<size_t>(swizzled_sf_bytes(M, kb)), stream);
            if (e != cudaSuccess) return e;
        }
        return launch_q_layout<true>(x, M, K, fmt, rule, g, q, sf, stream);
    }
    return launch_q_layout<false>(x, M, K, fmt, rule, g, q, sf, stream);
}

cudaError_t launch_fake_quantize(const void* x, int64_t M, int64_t K, int fmt, int rule, const float* g, void* y,
                                 cudaStream_t stream) {
    if (fmt == MXQ_NVFP4) return launch_fq<MXQ_NVFP4, 0>(x, M, K, g, y, stream);
    if (fmt == MXQ_MXFP8)
        return rule == MXQ_RULE_CEIL ? launch_fq<MXQ_MXFP8, MXQ_RULE_CEIL>(x, M, K, g, y, stream)
                                     : launch_fq<MXQ_MXFP8, MXQ_RULE_EVEN>(x, M, K, g, y, stream);
    return rule == MXQ_RULE_CEIL ? launch_fq<MXQ_MXFP4, MXQ_RULE_CEIL>(x, M, K, g, y, stream)
                                 : launch_fq<MXQ_MXFP4, MXQ_RULE_EVEN>(x, M, K, g, y, stream);
}

cudaError_t launch_quantize_running(const void* x, int64_t M, int64_t K, const float* amax_in, float* amax_out, void* q,
                                   void* sf, int layout, cudaStream_t stream) {
    // amax_out starts from the running state, then takes this batch's maximum
    cudaError_t e = cudaMemcpyAsync(amax_out, amax_in, sizeof(float), cudaMemcpyDeviceToDevice, stream);
    if (e != cudaSuccess) return e;
    if (layout == MXQ_SF_SWIZZLED) {
        const int64_t kb = K / 16;
        if (M % 128 != 0 || kb % 4 != 0) {
            e = cudaMemsetAsync(sf, 0, static_cast<size_t>(swizzled_sf_bytes(M, kb)), stream);
            if (e != cudaSuccess) return e;
        }
        return launch_q_running<true>(x, M, K, amax_in, amax_out, q, sf, stream);
    }
    return launch_q_running<false>(x, M, K, amax_in, amax_out, q, sf, stream);
}

cudaError_t launch_swizzle(const uint8_t* src, int64_t rows, int64_t kblocks, uint8_t* dst, cudaStream_t stream) {
    const int64_t total = swizzled_sf_bytes(rows, kblocks);
    int64_t blocks = ceil_div(total, 256);
    const int64_t cap = static_cast<int64_t>(sm_count()) * 16;
    if (blocks > cap) blocks = cap;
    swizzle_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        src, static_cast<uint32_t>(rows), static_cast<uint32_t>(kblocks), static_cast<uint32_t>(ceil_div(kblocks, 4)),
        dst, total);
    return cudaGetLastError();
}

cudaError_t launch_global_scale(const void* x, int64_t n, float* g_out, float* amax_out, cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(amax_out, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
    const int64_t n_chunks = n / 8;
    const int n_tail = static_cast<int>(n - n_chunks * 8);
    int64_t blocks = ceil_div(n_chunks > 0 ? n_chunks : 1, 256 * 4);
    const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    amax_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const uint4*>(x), n_chunks, static_cast<const uint16_t*>(x) + n_chunks * 8, n_tail,
        reinterpret_cast<unsigned int*>(amax_out));
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    global_scale_finalize<<<1, 1, 0, stream>>>(amax_out, g_out);
    return cudaGetLastError();
}

cudaError_t launch_selftest_timeout(uint64_t timeout_ns, cudaStream_t stream) {
    selftest_timeout_kernel<<<1, 32, 0, stream>>>(status_ptr(), timeout_ns);
    return cudaGetLastError();
}

}  // namespace mxq
