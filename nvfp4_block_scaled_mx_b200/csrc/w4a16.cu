// w4a16.cu -- weight-only (W4A16) GEMM: Out = A · dq(W)^T with bf16 activations A [M][K] and
// MXFP4 / NVFP4 weights W [N][K] (packed E2M1 codes, swizzled block scales), the serving mode of
// "Qwen3.5-27B-NVFP4-RTN-weight-only" (activations run bf16) and the Marlin mode of
// "Qwen3.5-27B-MXFP4-QAD-W4A4-LR1e-5-s1000" ("Evaluation results": one weight artifact serves
// W4A4 and W4A16).  The weights are the same bytes the W4A4 GEMM reads.
//
// One CTA per SM, persistent over BM x BN output tiles (BM = 128 * BMT), K in stages of 64:
//   warp 0      TMA producer: the bf16 A tile (128B-swizzled), the packed W codes (32 bytes per
//               row) and the W scale tiles of the stage
//   warp 1      TMEM owner; MMA issuer: tcgen05 kind::f16, bf16 x bf16 -> fp32, BMT accumulators
//   warps 2-5   dequantize W into bf16 directly in the 128B-swizzled B-operand layout (2-buffer
//               ring).  e2m1 * 2^e (MXFP4) and e2m1 * dec(s) (NVFP4) have at most 5 significant
//               bits, so the bf16 values are exact; g_W multiplies the fp32 accumulator instead.
//   warps 6-13  epilogue: drain the accumulators, scale by g_W (NVFP4), store bf16 or fp32
// The single-thread roles run as converged warps that issue through one elected lane.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "mxq_device.cuh"
#include "mxq_internal.h"

namespace mxq {
namespace {

constexpr int kW16DeqWarps = 4;
constexpr int kW16EpiWarps = 8;
constexpr int kW16Threads = (2 + kW16DeqWarps + kW16EpiWarps) * 32;

template <int FMT, int BMT, int BN>
struct W16Cfg {
    static constexpr int BM = 128 * BMT;
    static constexpr int BK = 64;  // K elements per stage: one 128-byte swizzle row of bf16 A
    static constexpr int STAGES = 3, BUFS = 2;
    static constexpr int BS = (FMT == MXQ_NVFP4) ? 16 : 32;
    static constexpr int A_BYTES = BM * 128;
    static constexpr int W_BYTES = BN * 32;
    static constexpr int SF_TILES = BN >= 128 ? BN / 128 : 1;  // 128-row scale tiles covering the tile's rows
    static constexpr int SF_BYTES = SF_TILES * 512;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_W = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SF = OFF_W + STAGES * W_BYTES;
    static constexpr int OFF_B = (OFF_SF + STAGES * SF_BYTES + 1023) / 1024 * 1024;
    static constexpr int OFF_BAR = OFF_B + BUFS * B_BYTES;
    static constexpr int N_BARS = 2 * STAGES + 2 * BUFS + 2;
    static constexpr int OFF_SLOT = OFF_BAR + N_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_SLOT + 16 + 1024;
    static constexpr uint32_t TMEM_COLS = BMT * BN <= 32 ? 32u : BMT * BN <= 64 ? 64u : BMT * BN <= 128 ? 128u
                                        : BMT * BN <= 256 ? 256u : 512u;
    static_assert(BMT * BN <= 512, "accumulators fit in TMEM");
    static_assert(BN % 64 == 0 && BN <= 256, "tile width");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct W16Args {
    const float* g_w;
    void* out;
    int M, N, K;
    int sf_col_tiles;  // ceil(K / bs / 4)
    int m_tiles, n_tiles, k_stages;
    uint32_t a_box_bytes;  // bytes of one A load (rows rounded up to 8, at most BM)
    int* status;
};

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

// The same on the integer and FMA pipes: the bf16 bit patterns of the E2M1 magnitudes 0, 0.5, 1,
// 1.5, 2, 3, 4, 6 come from byte-permute lookups (high and low byte tables, 3-bit selectors), the
// sign bits are moved to bit 15, and a bf16x2 multiply applies the scale s2 = (s, s).  Exact when
// every product is a normal bf16: the scale lies in [2^-125, 2^125] (MXFP4) or is an E4M3 value
// (NVFP4; products in [2^-10, 2688]).
__device__ __forceinline__ uint4 dequant8_prmt(uint32_t w, uint32_t s2) {
    constexpr uint32_t kHiLo = 0x3F3F3F00u, kHiHi = 0x40404040u;  // high bytes of magnitudes 0-3, 4-7
    constexpr uint32_t kLoLo = 0xC0800000u, kLoHi = 0xC0804000u;  // low bytes
    const uint32_t m0 = w & 0x7777u, m1 = (w >> 16) & 0x7777u;   // magnitudes as byte selectors
    uint32_t hi0 = __byte_perm(kHiLo, kHiHi, m0), lo0 = __byte_perm(kLoLo, kLoHi, m0);
    uint32_t hi1 = __byte_perm(kHiLo, kHiHi, m1), lo1 = __byte_perm(kLoLo, kLoHi, m1);
    // sign of code i (bit 4i + 3) to bit 7 of byte i: even codes come from sg << 4, odd codes from sg
    const uint32_t sg = w & 0x88888888u, sh = sg << 4;
    hi0 |= __byte_perm(sg, sh, 0x1504) & 0x80808080u;
    hi1 |= __byte_perm(sg, sh, 0x3726) & 0x80808080u;
    const uint32_t p[4] = {__byte_perm(lo0, hi0, 0x5140), __byte_perm(lo0, hi0, 0x7362), __byte_perm(lo1, hi1, 0x5140),
                           __byte_perm(lo1, hi1, 0x7362)};
    const __nv_bfloat162 sc = *reinterpret_cast<const __nv_bfloat162*>(&s2);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 v = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&p[i]), sc);
        o[i] = *reinterpret_cast<const uint32_t*>(&v);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int FMT, int BMT, int BN, bool OUT_F32>
__global__ void __launch_bounds__(kW16Threads, 1)
    w4a16_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_w,
                 const __grid_constant__ CUtensorMap tma_sf, const W16Args p) {
    using C = W16Cfg<FMT, BMT, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // A, W codes and scales landed
    uint64_t* empty = full + C::STAGES;                                // MMAs read A, dequant warps read W
    uint64_t* bready = empty + C::STAGES;                              // dequantized B buffer written
    uint64_t* bfree = bready + C::BUFS;                                // MMAs done with the B buffer
    uint64_t* accf = bfree + C::BUFS;                                  // accumulators ready
    uint64_t* acce = accf + 1;                                         // accumulators drained
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_SLOT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tma_a);
        prefetch_tmap(&tma_w);
        prefetch_tmap(&tma_sf);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + kW16DeqWarps);
        }
        for (int b = 0; b < C::BUFS; ++b) {
            mbar_init(&bready[b], kW16DeqWarps);
            mbar_init(&bfree[b], 1);
        }
        mbar_init(accf, 1);
        mbar_init(acce, kW16EpiWarps);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int num_tiles = p.m_tiles * p.n_tiles;
    if (warp == 0) {
        // TMA producer: the whole warp runs the loop; one elected lane issues
        const uint64_t pol_a = policy_evict_last();   // A tiles are reused by every N tile
        const uint64_t pol_w = policy_evict_first();  // W streams once per M sweep
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
            const int sf_tile0 = (nt * BN) >> 7;
            for (int ks = 0; ks < p.k_stages; ++ks) {
                if (!mbar_wait_warp(&empty[stage], phase ^ 1u, p.status, 41)) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    mbar_arrive_expect_tx(&full[stage], p.a_box_bytes + C::W_BYTES + C::SF_BYTES);
                    tma_load_2d(&tma_a, &full[stage], smem + C::OFF_A + stage * C::A_BYTES, ks * C::BK, mt * C::BM,
                                pol_a);
                    tma_load_2d(&tma_w, &full[stage], smem + C::OFF_W + stage * C::W_BYTES, ks * (C::BK / 2), nt * BN,
                                pol_w);
                    // the 512-byte scale tile holding this stage's blocks: 4 blocks of bs along K
                    const int kcol = (ks * C::BK / C::BS) >> 2;
#pragma unroll
                    for (int g = 0; g < C::SF_TILES; ++g)
                        tma_load_2d(&tma_sf, &full[stage], smem + C::OFF_SF + stage * C::SF_BYTES + g * 512, 0,
                                    ((sf_tile0 + g) * p.sf_col_tiles + kcol) * 2, pol_w);
                }
                __syncwarp();
                if (++stage == C::STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        // MMA issuer: the whole warp runs the loop; one elected lane issues
        const uint32_t idesc = mma_idesc_bf16(128, BN);
        int stage = 0, buf = 0;
        uint32_t phase = 0, bphase = 0, acc_phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            if (!mbar_wait_warp(acce, acc_phase ^ 1u, p.status, 42)) break;
            tc_fence_after();
            for (int ks = 0; ks < p.k_stages; ++ks) {
                if (!mbar_wait_warp(&full[stage], phase, p.status, 43) ||
                    !mbar_wait_warp(&bready[buf], bphase, p.status, 44)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_s = smem_u32(smem + C::OFF_A + stage * C::A_BYTES);
                const uint32_t b_s = smem_u32(smem + C::OFF_B + buf * C::B_BYTES);
                if (elect_one()) {
#pragma unroll
                    for (int j = 0; j < C::BK / 16; ++j) {
#pragma unroll
                        for (int h = 0; h < BMT; ++h)
                            mma_bf16(tmem_base + static_cast<uint32_t>(h * BN),
                                     smem_desc(a_s + h * 16384 + j * 32, 16, 1024, kLayoutSwizzle128B),
                                     smem_desc(b_s + j * 32, 16, 1024, kLayoutSwizzle128B), idesc, (ks | j) != 0 ? 1u : 0u);
                    }
                    tc_commit(&empty[stage]);
                    tc_commit(&bfree[buf]);
                }
                __syncwarp();
                if (++stage == C::STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
                if (++buf == C::BUFS) {
                    buf = 0;
                    bphase ^= 1u;
                }
            }
            if (!ok) break;
            if (elect_one()) tc_commit(accf);
            __syncwarp();
            acc_phase ^= 1u;
        }
    } else if (warp < 2 + kW16DeqWarps) {
        // dequantization: each thread converts BN / 64 items of 32 elements (one row half of the
        // stage, 16 bytes of codes); consecutive threads take consecutive rows, so the swizzled
        // 16-byte stores of a quarter warp hit 8 different bank groups
        constexpr int ITEMS = BN / 64;
        const int t = threadIdx.x - 64;
        int stage = 0, buf = 0;
        uint32_t phase = 0, bphase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            const int nt = tile / p.m_tiles;
            for (int ks = 0; ks < p.k_stages; ++ks) {
                if (!mbar_wait_warp(&full[stage], phase, p.status, 45) ||
                    !mbar_wait_warp(&bfree[buf], bphase ^ 1u, p.status, 46)) {
                    ok = false;
                    break;
                }
                const uint32_t w_s = smem_u32(smem + C::OFF_W + stage * C::W_BYTES);
                const uint32_t sf_s = smem_u32(smem + C::OFF_SF + stage * C::SF_BYTES);
                uint4 codes[ITEMS];
                uint32_t sc[ITEMS];
#pragma unroll
                for (int i = 0; i < ITEMS; ++i) {
                    const int id = t + 128 * i;
                    const int row = id % BN, half = id / BN;
                    codes[i] = ld_shared_v4(w_s + row * 32 + half * 16);
                    const int r_abs = nt * BN + row;
                    const int g = (r_abs >> 7) - ((nt * BN) >> 7), rr = r_abs & 127;
                    const int kb = ks * (C::BK / C::BS) + half * (32 / C::BS);  // first block of the item
                    const uint32_t off = g * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (kb & 3);
                    sc[i] = (FMT == MXQ_NVFP4) ? ld_shared_u16(sf_s + off) : ld_shared_u8(sf_s + off);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[stage]);  // this warp is done with the stage's W bytes
                const uint32_t b_s = smem_u32(smem + C::OFF_B + buf * C::B_BYTES);
#pragma unroll
                for (int i = 0; i < ITEMS; ++i) {
                    const int id = t + 128 * i;
                    const int row = id % BN, half = id / BN;
                    const uint32_t rbase = b_s + row * 128;
                    const uint32_t sw = static_cast<uint32_t>(row & 7);
                    uint4 o0, o1, o2, o3;
                    if constexpr (FMT == MXQ_NVFP4) {
                        // E4M3 block scales (exact in bf16); the first 16 elements take s0, the rest s1
                        const uint32_t c0 = sc[i] & 0xFFu, c1 = sc[i] >> 8;
                        const __nv_bfloat16 b0 = __float2bfloat16_rn(e4m3_decode_pos(c0 & 0x7Fu) * ((c0 & 0x80u) ? -1.0f : 1.0f));
                        const __nv_bfloat16 b1 = __float2bfloat16_rn(e4m3_decode_pos(c1 & 0x7Fu) * ((c1 & 0x80u) ? -1.0f : 1.0f));
                        const uint32_t u0 = *reinterpret_cast<const uint16_t*>(&b0), u1 = *reinterpret_cast<const uint16_t*>(&b1);
                        o0 = dequant8_prmt(codes[i].x, u0 * 0x10001u);
                        o1 = dequant8_prmt(codes[i].y, u0 * 0x10001u);
                        o2 = dequant8_prmt(codes[i].z, u1 * 0x10001u);
                        o3 = dequant8_prmt(codes[i].w, u1 * 0x10001u);
                    } else {
                        const int e = static_cast<int>(sc[i]) - 127;
                        if (e >= -125 && e <= 125) {
                            const uint32_t s2 = (static_cast<uint32_t>(e + 127) << 7) * 0x10001u;  // bf16 2^e, twice
                            o0 = dequant8_prmt(codes[i].x, s2);
                            o1 = dequant8_prmt(codes[i].y, s2);
                            o2 = dequant8_prmt(codes[i].z, s2);
                            o3 = dequant8_prmt(codes[i].w, s2);
                        } else {
                            const float s = pow2f(e);
                            o0 = dequant8_cvt(codes[i].x, s);
                            o1 = dequant8_cvt(codes[i].y, s);
                            o2 = dequant8_cvt(codes[i].z, s);
                            o3 = dequant8_cvt(codes[i].w, s);
                        }
                    }
                    st_shared_v4(rbase + (((4 * half + 0) ^ sw) << 4), o0);
                    st_shared_v4(rbase + (((4 * half + 1) ^ sw) << 4), o1);
                    st_shared_v4(rbase + (((4 * half + 2) ^ sw) << 4), o2);
                    st_shared_v4(rbase + (((4 * half + 3) ^ sw) << 4), o3);
                }
                fence_proxy_async_smem();  // generic-proxy stores, read next by the tensor cores
                __syncwarp();
                if (lane == 0) mbar_arrive(&bready[buf]);
                if (++stage == C::STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
                if (++buf == C::BUFS) {
                    buf = 0;
                    bphase ^= 1u;
                }
            }
        }
    } else {
        // epilogue: warp e drains TMEM sub-partition (warp % 4) of accumulator h, columns [c0, c0 + NC)
        const int e = warp - 2 - kW16DeqWarps;
        const int sub = warp & 3;
        const int h = (BMT == 2) ? (e >> 2) : 0;
        constexpr int NC = (BMT == 2) ? BN : BN / 2;
        const int c0 = (BMT == 2) ? 0 : (e >> 2) * NC;
        const float alpha = (FMT == MXQ_NVFP4) ? *p.g_w : 1.0f;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
            if (!mbar_wait(accf, acc_phase, p.status, 47)) break;
            tc_fence_after();
            const int m = mt * C::BM + h * 128 + sub * 32 + lane;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + static_cast<uint32_t>(h * BN + c0);
#pragma unroll 1
            for (int c = 0; c < NC; c += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(t_row + c, r);
                tmem_ld_wait();
                const int nb = nt * BN + c0 + c;
                if (m < p.M && nb < p.N) {
                    if constexpr (OUT_F32) {
                        float* orow = static_cast<float*>(p.out) + static_cast<int64_t>(m) * p.N;
                        if ((p.N & 3) == 0 && nb + 32 <= p.N) {
                            float4* dst = reinterpret_cast<float4*>(orow + nb);
#pragma unroll
                            for (int v = 0; v < 8; ++v)
                                dst[v] = make_float4(__fmul_rn(__uint_as_float(r[4 * v]), alpha),
                                                     __fmul_rn(__uint_as_float(r[4 * v + 1]), alpha),
                                                     __fmul_rn(__uint_as_float(r[4 * v + 2]), alpha),
                                                     __fmul_rn(__uint_as_float(r[4 * v + 3]), alpha));
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (nb + i < p.N) orow[nb + i] = __fmul_rn(__uint_as_float(r[i]), alpha);
                        }
                    } else {
                        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(m) * p.N;
                        uint32_t packed[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const __nv_bfloat162 b = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[2 * i]), alpha),
                                                                           __fmul_rn(__uint_as_float(r[2 * i + 1]), alpha));
                            packed[i] = *reinterpret_cast<const uint32_t*>(&b);
                        }
                        if ((p.N & 7) == 0 && nb + 32 <= p.N) {
                            uint4* dst = reinterpret_cast<uint4*>(orow + nb);
#pragma unroll
                            for (int v = 0; v < 4; ++v)
                                dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
                        } else {
                            uint16_t* o16 = reinterpret_cast<uint16_t*>(orow);
#pragma unroll
                            for (int v = 0; v < 16; ++v) {
                                if (nb + 2 * v < p.N) o16[nb + 2 * v] = static_cast<uint16_t>(packed[v] & 0xFFFFu);
                                if (nb + 2 * v + 1 < p.N) o16[nb + 2 * v + 1] = static_cast<uint16_t>(packed[v] >> 16);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce);
            acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// bf16 A [M][K]: boxes of 64 elements (128 bytes) x box_rows, 128B swizzle.
bool make_a16_map(CUtensorMap* m, const void* A, int64_t M, int64_t K, uint32_t box_rows) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(A), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// packed FP4 W [N][K/2]: boxes of 32 bytes (64 elements) x box_rows, no swizzle.
bool make_w4_map(CUtensorMap* m, const void* W, int64_t N, int64_t K, uint32_t box_rows) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    cuuint32_t box[2] = {32, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(W), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Swizzled W scales as rows of 256 bytes (two per 512-byte tile); a box is one tile.
bool make_w_sf_map(CUtensorMap* m, const void* sf, int64_t rows, int64_t kblocks) {
    auto enc = encode_fn();
    if (!enc) return false;
    const uint64_t half_rows = static_cast<uint64_t>(swizzled_sf_bytes(rows, kblocks) / 256);
    cuuint64_t dims[2] = {256, half_rows};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {256, 2};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(sf), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT, int BMT, int BN, bool F32>
int run_w16(const void* A, const void* Wq, const uint8_t* Wsf, const float* g_w, int64_t M, int64_t N, int64_t K,
            void* out, cudaStream_t stream) {
    using C = W16Cfg<FMT, BMT, BN>;
    auto kern = w4a16_kernel<FMT, BMT, BN, F32>;
    const uint32_t a_rows = static_cast<uint32_t>(M >= C::BM ? C::BM : ceil_div(M, 8) * 8);
    CUtensorMap ta, tw, tsf;
    if (!make_a16_map(&ta, A, M, K, a_rows) || !make_w4_map(&tw, Wq, N, K, BN) ||
        !make_w_sf_map(&tsf, Wsf, N, K / C::BS))
        return MXQ_ERR_CUDA;
    W16Args args = {};
    args.g_w = g_w;
    args.out = out;
    args.M = static_cast<int>(M);
    args.N = static_cast<int>(N);
    args.K = static_cast<int>(K);
    args.sf_col_tiles = static_cast<int>(ceil_div(K / C::BS, 4));
    args.m_tiles = static_cast<int>(ceil_div(M, C::BM));
    args.n_tiles = static_cast<int>(ceil_div(N, BN));
    args.k_stages = static_cast<int>(K / C::BK);
    args.a_box_bytes = a_rows * 128;
    args.status = status_ptr();
    int dev = 0;
    cudaGetDevice(&dev);
    static bool attr_done[64] = {};
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
            return MXQ_ERR_CUDA;
        attr_done[dev] = true;
    }
    const int64_t tiles = static_cast<int64_t>(args.m_tiles) * args.n_tiles;
    const int grid = static_cast<int>(tiles < sm_count() ? tiles : sm_count());
    kern<<<grid, kW16Threads, C::SMEM_BYTES, stream>>>(ta, tw, tsf, args);
    return cudaGetLastError() == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

template <int FMT, bool F32>
int dispatch_w16(const void* A, const void* Wq, const uint8_t* Wsf, const float* g_w, int64_t M, int64_t N,
                 int64_t K, void* out, cudaStream_t stream) {
    // More than 128 rows: 256 x 256 tiles, two M=128 MMAs sharing each dequantized W tile.  Up to
    // 128 rows: 128 x 64 tiles, which gives the most CTAs for the weight stream.
    if (M > 128) return run_w16<FMT, 2, 256, F32>(A, Wq, Wsf, g_w, M, N, K, out, stream);
    return run_w16<FMT, 1, 64, F32>(A, Wq, Wsf, g_w, M, N, K, out, stream);
}

}  // namespace

int launch_w4a16(const void* A, const void* W_q, const uint8_t* W_sf, const float* g_W, int64_t M, int64_t N,
                 int64_t K, int fmt, int out_type, void* out, cudaStream_t stream) {
    const bool f32 = out_type == MXQ_OUT_FP32;
    if (fmt == MXQ_NVFP4)
        return f32 ? dispatch_w16<MXQ_NVFP4, true>(A, W_q, W_sf, g_W, M, N, K, out, stream)
                   : dispatch_w16<MXQ_NVFP4, false>(A, W_q, W_sf, g_W, M, N, K, out, stream);
    return f32 ? dispatch_w16<MXQ_MXFP4, true>(A, W_q, W_sf, g_W, M, N, K, out, stream)
               : dispatch_w16<MXQ_MXFP4, false>(A, W_q, W_sf, g_W, M, N, K, out, stream);
}

}  // namespace mxq
