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

#include "dequant.cuh"
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
    static constexpr int STG_BYTES = 32 * 64;  // per epilogue warp: 32 rows x 32 bf16 columns (64B swizzle)
    static constexpr int OFF_STG = OFF_B + BUFS * B_BYTES;
    static constexpr int OFF_BAR = OFF_STG + kW16EpiWarps * STG_BYTES;
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
    int tma_store;         // bf16 output through TMA stores (rows of N * 2 bytes are 16-byte multiples)
    int* status;
};


// f2 for an NVFP4 block with E4M3 code c: 2^118 times the code's value, so that the dequantized
// elements are 2^-8 times the NVFP4 values (the epilogue multiplies by 2^8).  The factor lies in
// [2^109, 2^127) and the products in [2^-18, 10.5]: all exact normal bf16 numbers.
__device__ __forceinline__ uint32_t nvfp4_factor2(uint32_t c) {
    const float f = e4m3_decode_pos(c & 0x7Fu) * 0x1p118f;
    const __nv_bfloat16 h = __float2bfloat16_rn((c & 0x80u) ? -f : f);
    return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&h)) * 0x10001u;
}

// Scale applied after the fp32 accumulation: NVFP4 takes back the 2^-8 of its dequantization
// factor (an exact power-of-two step) before the global scale.
template <int FMT>
__device__ __forceinline__ float w16_epilogue(float acc, float g) {
    return (FMT == MXQ_NVFP4) ? __fmul_rn(__fmul_rn(acc, 256.0f), g) : acc;
}

// True if the E8M0 codes in the low `n` bytes of `codes` all lie in [2, 128] (scales 2^-125 .. 2),
// where dequant8_mul is exact.
__device__ __forceinline__ bool mx_scales_in_range(uint32_t codes, int n) {
    bool ok = true;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (i < n) {
            const uint32_t b = (codes >> (8 * i)) & 0xFFu;
            ok = ok && b >= 2u && b <= 128u;
        }
    return ok;
}

template <int FMT, int BMT, int BN, bool OUT_F32>
__global__ void __launch_bounds__(kW16Threads, 1)
    w4a16_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_w,
                 const __grid_constant__ CUtensorMap tma_sf, const __grid_constant__ CUtensorMap tma_out,
                 const W16Args p) {
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
        if (!OUT_F32 && p.tma_store) prefetch_tmap(&tma_out);
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
    pdl_wait();  // launched with programmatic serialization: inputs are read, outputs written after this
    pdl_launch_dependents();  // the next kernel on the stream may start its prologue

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
                    const int row = id >> 1, half = id & 1;  // a warp reads 512 contiguous bytes of codes
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
                // MXFP4: the multiply path unless some scale of the warp's items leaves 2^-125 .. 2
                bool fast = true;
                if constexpr (FMT != MXQ_NVFP4) {
                    bool mine = true;
#pragma unroll
                    for (int i = 0; i < ITEMS; ++i) mine = mine && mx_scales_in_range(sc[i], 1);
                    fast = __all_sync(0xFFFFFFFFu, mine);
                }
#pragma unroll
                for (int i = 0; i < ITEMS; ++i) {
                    const int id = t + 128 * i;
                    const int row = id >> 1, half = id & 1;  // a warp reads 512 contiguous bytes of codes
                    const uint32_t rbase = b_s + row * 128;
                    const uint32_t sw = static_cast<uint32_t>(row & 7);
                    uint4 o0, o1, o2, o3;
                    if constexpr (FMT == MXQ_NVFP4) {
                        // E4M3 block scales; the first 16 elements take s0, the rest s1
                        const uint32_t f0 = nvfp4_factor2(sc[i] & 0xFFu), f1 = nvfp4_factor2(sc[i] >> 8);
                        o0 = dequant8_mul(codes[i].x, f0);
                        o1 = dequant8_mul(codes[i].y, f0);
                        o2 = dequant8_mul(codes[i].z, f1);
                        o3 = dequant8_mul(codes[i].w, f1);
                    } else if (fast) {
                        const uint32_t f = mx_factor2(sc[i]);
                        o0 = dequant8_mul(codes[i].x, f);
                        o1 = dequant8_mul(codes[i].y, f);
                        o2 = dequant8_mul(codes[i].z, f);
                        o3 = dequant8_mul(codes[i].w, f);
                    } else {
                        const float s = pow2f(static_cast<int>(sc[i]) - 127);
                        o0 = dequant8_cvt(codes[i].x, s);
                        o1 = dequant8_cvt(codes[i].y, s);
                        o2 = dequant8_cvt(codes[i].z, s);
                        o3 = dequant8_cvt(codes[i].w, s);
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
            if (!OUT_F32 && p.tma_store) {
                // 32 x 32 bf16 tiles through this warp's staging buffer (64B swizzle: 16-byte piece q
                // of row r at piece q ^ ((r >> 1) & 3)) and one TMA store each, clipped at the M and N
                // edges; the accumulator is released right after its last columns are in registers
                uint8_t* stg = smem + C::OFF_STG + e * C::STG_BYTES;
                const uint32_t st_row = smem_u32(stg) + lane * 64;
                const uint32_t sw = static_cast<uint32_t>((lane >> 1) & 3);
#pragma unroll 1
                for (int c = 0; c < NC; c += 32) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(t_row + c, r);
                    tmem_ld_wait();
                    if (c + 32 == NC) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(acce);
                    }
                    uint32_t packed[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const __nv_bfloat162 b = __floats2bfloat162_rn(w16_epilogue<FMT>(__uint_as_float(r[2 * i]), alpha),
                                                                       w16_epilogue<FMT>(__uint_as_float(r[2 * i + 1]), alpha));
                        packed[i] = *reinterpret_cast<const uint32_t*>(&b);
                    }
                    if (lane == 0) bulk_wait_group_read0();  // the staging tile is free again
                    __syncwarp();
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        st_shared_v4(st_row + ((q ^ sw) << 4),
                                     make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]));
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tma_out, stg, nt * BN + c0 + c, mt * C::BM + h * 128 + sub * 32);
                        bulk_commit_group();
                    }
                }
                acc_phase ^= 1u;
                continue;
            }
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
                                dst[v] = make_float4(w16_epilogue<FMT>(__uint_as_float(r[4 * v]), alpha),
                                                     w16_epilogue<FMT>(__uint_as_float(r[4 * v + 1]), alpha),
                                                     w16_epilogue<FMT>(__uint_as_float(r[4 * v + 2]), alpha),
                                                     w16_epilogue<FMT>(__uint_as_float(r[4 * v + 3]), alpha));
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (nb + i < p.N) orow[nb + i] = w16_epilogue<FMT>(__uint_as_float(r[i]), alpha);
                        }
                    } else {
                        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(m) * p.N;
                        uint32_t packed[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const __nv_bfloat162 b = __floats2bfloat162_rn(w16_epilogue<FMT>(__uint_as_float(r[2 * i]), alpha),
                                                                           w16_epilogue<FMT>(__uint_as_float(r[2 * i + 1]), alpha));
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
        if (!OUT_F32 && p.tma_store && lane == 0) bulk_wait_group0();  // the output has left shared memory
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ weights dequantized into TMEM
//
// For few tokens (M <= 128) the weights dominate the traffic.  Here Out^T tile = W tile [128 weight
// rows] x A tile^T [NT tokens]: the MMA's A operand is the dequantized weight tile, which the
// dequant warps write straight into TMEM (tcgen05.st: a thread's TMEM lane is its weight row), and
// its B operand is the bf16 activation tile in shared memory.  K advances 256 per stage, so each
// weight row contributes a full 128-byte line per stage (the 128 rows arrive as one 16 KB TMA box
// with a 128-byte swizzle).
//   warp 0       TMA producer: 4 activation boxes (NT tokens x 64 K, 128B-swizzled), 128 rows of
//                packed codes (128 bytes each), their scale tiles
//   warp 1       TMEM owner; MMA issuer (A from TMEM, B from shared memory), 16 MMAs per stage
//   warps 2-9    dequantization into TMEM slots of 128 columns: two warps per sub-partition, each
//                converting 128 of the stage's 256 K elements of its 32 rows
//   warps 10-17  epilogue: a lane owns one weight row (output column), so a warp's store for one
//                token covers 32 consecutive output columns
// SPLIT: a cluster of k_split CTAs shares one tile, each CTA a contiguous range of K stages, and
// the partials are reduced through distributed shared memory in the leader.  Otherwise the grid is
// persistent over tiles (tokens fastest) with two accumulators when TMEM has room.

constexpr int kWtDeqWarps = 8;  // 16 (the epilogue warps too) when every CTA owns one tile
constexpr int kWtGroups16 = 2;  // 16 dequantizing warps form this many groups taking turns on stages
constexpr int kWtEpiWarps = 8;
constexpr int kWtThreads = (2 + kWtDeqWarps + kWtEpiWarps) * 32;
constexpr int kWtK = 256;  // K elements per stage

template <int FMT, int NT, int STAGES, int AS, bool SPLIT>
struct W16TCfg {
    static constexpr int BS = (FMT == MXQ_NVFP4) ? 16 : 32;
    static constexpr int SF_ATOMS = kWtK / BS / 4;           // 512-byte scale tiles per stage (2 or 4)
    static constexpr int ACT_SUB = NT * 128;                 // one activation box: NT rows x 128 bytes
    static constexpr int ACT_BYTES = 4 * ACT_SUB;
    static constexpr int W_BYTES = 128 * 128;
    static constexpr int SF_BYTES = SF_ATOMS * 512;
    static constexpr int ACC = (!SPLIT && 2 * NT + AS * 128 <= 512) ? 2 : 1;
    static constexpr int A_TMEM = ACC * NT;  // first column of the weight slots
    static constexpr int COLS_USED = A_TMEM + AS * 128;
    static constexpr uint32_t TMEM_COLS = COLS_USED <= 256 ? 256u : 512u;
    static constexpr int OFF_ACT = 0;
    static constexpr int OFF_W = OFF_ACT + STAGES * ACT_BYTES;
    static constexpr int OFF_SF = OFF_W + STAGES * W_BYTES;
    // SPLIT at NT = 32: the partials of up to 3 other CTAs (16 KB each) get a buffer of their own, so
    // that the other CTAs send them as soon as their MMAs are done; otherwise (NT = 64, 32 KB each)
    // they reuse the leader's operand ring once the leader signals that its MMAs are done
    static constexpr bool RED_OWN = SPLIT && NT == 32;
    static constexpr int OFF_RED = OFF_SF + STAGES * SF_BYTES;
    static constexpr int RED_BYTES = RED_OWN ? 3 * 128 * NT * 4 : 0;
    static constexpr int OFF_BAR = OFF_RED + RED_BYTES;
    static constexpr int N_BARS = 2 * STAGES + 2 * AS + 2 * ACC + 2;
    static constexpr int OFF_SLOT = OFF_BAR + N_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_SLOT + 16 + 1024;
    static_assert(NT % 16 == 0 && NT >= 16 && NT <= 256, "MMA N");
    static_assert(COLS_USED <= 512, "TMEM budget");
    static_assert(!SPLIT || RED_OWN || 3 * 128 * NT * 4 <= OFF_RED, "split-K partials fit in the operand ring");
    static_assert(ACT_SUB % 1024 == 0, "128B-swizzled activation boxes stay 1024-byte aligned");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct W16TArgs {
    const float* g_w;
    void* out;
    int M, N, K;
    int sf_col_tiles;
    int t_tiles, w_tiles, k_stages;
    uint32_t k_split;
    uint32_t act_box_bytes;
    int* status;
};

template <int FMT, int NT, int STAGES, int AS, bool SPLIT, int DQW, bool OUT_F32>
__global__ void __launch_bounds__(kWtThreads, 1)
    w4a16_tmem_kernel(const __grid_constant__ CUtensorMap tma_act, const __grid_constant__ CUtensorMap tma_w,
                      const __grid_constant__ CUtensorMap tma_sf, const W16TArgs p) {
    using C = W16TCfg<FMT, NT, STAGES, AS, SPLIT>;
    constexpr int GROUPS = DQW == 16 ? kWtGroups16 : 1;  // dequantizing warp groups, taking turns on stages
    constexpr int WPS = DQW / GROUPS;                    // dequantizing warps per stage
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // activations, codes, scales landed
    uint64_t* empty = full + STAGES;                                   // MMAs read activations, dequant read codes
    uint64_t* aready = empty + STAGES;                                 // weight slot written
    uint64_t* aempty = aready + AS;                                    // MMAs done with the weight slot
    uint64_t* accf = aempty + AS;                                      // accumulator ready
    uint64_t* acce = accf + C::ACC;                                    // accumulator drained
    uint64_t* rready = acce + C::ACC;  // split, non-leaders: the leader's operand ring is free for the partials
    uint64_t* rfull = rready + 1;      // split, leader: every partial has landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_SLOT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t split = 0, splits = 1;
    if constexpr (SPLIT) {
        split = cluster_ctarank();
        splits = p.k_split;
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tma_act);
        prefetch_tmap(&tma_w);
        prefetch_tmap(&tma_sf);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + WPS);
        }
        for (int a = 0; a < AS; ++a) {
            mbar_init(&aready[a], WPS);
            mbar_init(&aempty[a], 1);
        }
        for (int b = 0; b < C::ACC; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], kWtEpiWarps);
        }
        if constexpr (SPLIT) {
            mbar_init(rready, 1);
            mbar_init(rfull, 1);
            // the other splits-1 CTAs' partial tiles, counted in bytes
            if (split == 0) mbar_arrive_expect_tx(rfull, (splits - 1) * 128u * NT * 4u);
        }
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if constexpr (SPLIT) cluster_arrive_relaxed();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();  // launched with programmatic serialization: inputs are read, outputs written after this
    pdl_launch_dependents();  // the next kernel on the stream may start its prologue

    // tiles: tokens fastest; a SPLIT cluster takes one tile and a contiguous range of K stages
    const int num_tiles = p.t_tiles * p.w_tiles;
    const int first = SPLIT ? static_cast<int>(blockIdx.x / splits) : static_cast<int>(blockIdx.x);
    const int step = SPLIT ? num_tiles : static_cast<int>(gridDim.x);
    const int per = (p.k_stages + static_cast<int>(splits) - 1) / static_cast<int>(splits);
    const int k0 = static_cast<int>(split) * per;
    const int k1 = min(p.k_stages, k0 + per);

    if (warp == 0) {
        const uint64_t pol_act = policy_evict_last();  // activation tiles are reused by every weight tile
        const uint64_t pol_w = policy_evict_first();   // weights stream
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = first; tile < num_tiles && ok; tile += step) {
            const int tt = tile % p.t_tiles, wt = tile / p.t_tiles;
            for (int ks = k0; ks < k1; ++ks) {
                if (!mbar_wait_warp(&empty[stage], phase ^ 1u, p.status, 51)) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    mbar_arrive_expect_tx(&full[stage], 4 * p.act_box_bytes + C::W_BYTES + C::SF_BYTES);
                    uint8_t* act = smem + C::OFF_ACT + stage * C::ACT_BYTES;
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        tma_load_2d(&tma_act, &full[stage], act + b * C::ACT_SUB, ks * kWtK + b * 64, tt * NT, pol_act);
                    tma_load_2d(&tma_w, &full[stage], smem + C::OFF_W + stage * C::W_BYTES, ks * (kWtK / 2), wt * 128,
                                pol_w);
                    // the stage's SF_ATOMS consecutive 512-byte scale tiles of these 128 rows
                    tma_load_2d(&tma_sf, &full[stage], smem + C::OFF_SF + stage * C::SF_BYTES, 0,
                                (wt * p.sf_col_tiles + ks * C::SF_ATOMS) * 2, pol_w);
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        const uint32_t idesc = mma_idesc_bf16(128, NT);
        int stage = 0, slot = 0, acc = 0;
        uint32_t phase = 0, sphase = 0, acc_phase = 0;
        bool ok = true;
        for (int tile = first; tile < num_tiles && ok; tile += step) {
            if (!mbar_wait_warp(&acce[acc], acc_phase ^ 1u, p.status, 52)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * NT);
            for (int ks = k0; ks < k1; ++ks) {
                if (!mbar_wait_warp(&full[stage], phase, p.status, 53) ||
                    !mbar_wait_warp(&aready[slot], sphase, p.status, 54)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t act_s = smem_u32(smem + C::OFF_ACT + stage * C::ACT_BYTES);
                const uint32_t a_tmem = tmem_base + static_cast<uint32_t>(C::A_TMEM + slot * 128);
                if (elect_one()) {
#pragma unroll
                    for (int j = 0; j < kWtK / 16; ++j)
                        mma_bf16_ts(d_tmem, a_tmem + j * 8,
                                    smem_desc(act_s + (j >> 2) * C::ACT_SUB + (j & 3) * 32, 16, 1024, kLayoutSwizzle128B),
                                    idesc, (ks > k0 || j > 0) ? 1u : 0u);
                    tc_commit(&empty[stage]);
                    tc_commit(&aempty[slot]);
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
                if (++slot == AS) {
                    slot = 0;
                    sphase ^= 1u;
                }
            }
            if (!ok) break;
            if (elect_one()) tc_commit(&accf[acc]);
            __syncwarp();
            if (++acc == C::ACC) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    } else if (warp < 2 + DQW) {
        // dequantization: this thread's weight row of the tile is its TMEM lane; in the stages of
        // its group, warp quad kq converts K elements [KE * kq, + KE) (KE / 2 bytes of codes, NBLK
        // scale blocks) into TMEM columns [KE / 2 * kq, + KE / 2) of the slot, 64 elements at a time.
        // Groups taking turns keep one group's shared-memory loads and waits under another's math.
        constexpr int KE = 4 * kWtK / WPS;   // 128 or 64
        constexpr int NCH = KE / 32;         // 16-byte code pieces per thread
        constexpr int NBLK = KE / C::BS;     // scale blocks per thread
        constexpr int NSW = (NBLK + 3) / 4;  // 32-bit scale words per thread
        const int r = 32 * (warp & 3) + lane;
        const int kq = ((warp - 2) % WPS) >> 2;
        const int grp = (warp - 2) / WPS;
        const int blk0 = NBLK * kq;  // the warp's first scale block in the stage
        int turn = 0;
        const uint32_t lane_addr = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        const uint32_t sw = static_cast<uint32_t>(r & 7);  // 128-byte swizzle of the code rows
        int stage = 0, slot = 0;
        uint32_t phase = 0, sphase = 0;
        bool ok = true;
        for (int tile = first; tile < num_tiles && ok; tile += step) {
            for (int ks = k0; ks < k1; ++ks) {
                const bool mine = GROUPS == 1 || turn == grp;
                if (++turn == GROUPS) turn = 0;
                if (mine) {
                    if (!mbar_wait_warp(&full[stage], phase, p.status, 55)) {
                        ok = false;
                        break;
                    }
                    const uint32_t w_row = smem_u32(smem + C::OFF_W + stage * C::W_BYTES) + r * 128;
                    uint4 c[NCH];
#pragma unroll
                    for (int q = 0; q < NCH; ++q) c[q] = ld_shared_v4(w_row + (((NCH * kq + q) ^ sw) << 4));
                    // a 512-byte scale tile holds 4 consecutive blocks of each of the 128 rows
                    const uint32_t sf_row = smem_u32(smem + C::OFF_SF + stage * C::SF_BYTES) + (r & 31) * 16 + (r >> 5) * 4;
                    uint32_t sc[NSW];
#pragma unroll
                    for (int i = 0; i < NSW; ++i)
                        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(sc[i]) : "r"(sf_row + ((blk0 >> 2) + i) * 512));
                    if constexpr (NBLK < 4) sc[0] >>= 8 * (blk0 & 3);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[stage]);  // this warp is done with the stage's codes and scales
                    if (!mbar_wait_warp(&aempty[slot], sphase ^ 1u, p.status, 56)) {
                        ok = false;
                        break;
                    }
                    const uint32_t t_col =
                        tmem_base + lane_addr + static_cast<uint32_t>(C::A_TMEM + slot * 128 + kq * (KE / 2));
                    // MXFP4: the multiply path unless some scale of the warp leaves 2^-125 .. 2
                    const bool fast = (FMT == MXQ_NVFP4) || __all_sync(0xFFFFFFFFu, mx_scales_in_range(sc[0], NBLK));
                    if (fast) {
                        uint32_t f2[NBLK];  // per-block dequantization factors
#pragma unroll
                        for (int b = 0; b < NBLK; ++b) {
                            const uint32_t code = (sc[b >> 2] >> (8 * (b & 3))) & 0xFFu;
                            f2[b] = (FMT == MXQ_NVFP4) ? nvfp4_factor2(code) : mx_factor2(code);
                        }
#pragma unroll
                        for (int hq = 0; hq < KE / 64; ++hq) {  // 64 elements (two 16-byte code pieces) at a time
                            uint32_t v[32];
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int wi = 8 * hq + j;  // word index in this warp's KE elements
                                const uint4 cc = c[wi >> 2];
                                const uint32_t word = (wi & 3) == 0 ? cc.x : (wi & 3) == 1 ? cc.y : (wi & 3) == 2 ? cc.z : cc.w;
                                const uint4 o = dequant8_mul(word, f2[wi * 8 / C::BS]);
                                v[4 * j + 0] = o.x;
                                v[4 * j + 1] = o.y;
                                v[4 * j + 2] = o.z;
                                v[4 * j + 3] = o.w;
                            }
                            tmem_st_cols<32>(t_col + hq * 32, v);
                        }
                    } else {
#pragma unroll
                        for (int hq = 0; hq < KE / 64; ++hq) {
                            uint32_t v[32];
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int wi = 8 * hq + j;
                                const uint4 cc = c[wi >> 2];
                                const uint32_t word = (wi & 3) == 0 ? cc.x : (wi & 3) == 1 ? cc.y : (wi & 3) == 2 ? cc.z : cc.w;
                                const uint32_t code = (sc[0] >> (8 * (wi >> 2))) & 0xFFu;
                                const uint4 o = dequant8_cvt(word, pow2f(static_cast<int>(code) - 127));
                                v[4 * j + 0] = o.x;
                                v[4 * j + 1] = o.y;
                                v[4 * j + 2] = o.z;
                                v[4 * j + 3] = o.w;
                            }
                            tmem_st_cols<32>(t_col + hq * 32, v);
                        }
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&aready[slot]);
                }
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
                if (++slot == AS) {
                    slot = 0;
                    sphase ^= 1u;
                }
            }
        }
    }

    // epilogue: warp e drains TMEM sub-partition (warp % 4), i.e. weight rows 32 * sub .. + 31, and
    // token columns [half * NT / 2, + NT / 2) of the tile
    constexpr int HC = NT / 2;
    const bool epi = warp >= 2 + kWtDeqWarps;
    const int sub = warp & 3;
    const int half = (warp - 2 - kWtDeqWarps) >> 2;
    const float alpha = (FMT == MXQ_NVFP4) ? *p.g_w : 1.0f;
    auto store = [&](int tt, int wt, int j, float val) {
        const int tok = tt * NT + half * HC + j, n = wt * 128 + sub * 32 + lane;
        if (tok < p.M && n < p.N) {
            const float y = w16_epilogue<FMT>(val, alpha);
            if constexpr (OUT_F32)
                static_cast<float*>(p.out)[static_cast<int64_t>(tok) * p.N + n] = y;
            else
                static_cast<__nv_bfloat16*>(p.out)[static_cast<int64_t>(tok) * p.N + n] = __float2bfloat16_rn(y);
        }
    };
    if constexpr (!SPLIT) {
        if (epi) {
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int tile = first; tile < num_tiles; tile += step) {
                const int tt = tile % p.t_tiles, wt = tile / p.t_tiles;
                if (!mbar_wait(&accf[acc], acc_phase, p.status, 57)) break;
                tc_fence_after();
                const uint32_t t_row =
                    tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + static_cast<uint32_t>(acc * NT + half * HC);
#pragma unroll 1
                for (int c = 0; c < HC; c += 16) {
                    uint32_t rr[16];
                    tmem_ld_32x32b_x16(t_row + c, rr);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; ++j) store(tt, wt, c + j, __uint_as_float(rr[j]));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce[acc]);
                if (++acc == C::ACC) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
        }
        tc_fence_before();
        __syncthreads();
    } else {
        // every CTA's epilogue warps take their partial tile into registers.  The others send their
        // partials with st.async, counted in bytes on the leader's barrier, and leave: at NT = 32
        // into a buffer of the leader's own at once (the hand-shake below cost about 0.9 us between
        // the leader's last MMAs and the partials leaving), at NT = 64 into the leader's operand
        // ring once the leader has freed it (a remote arrive per other CTA).  Layout in
        // the leader: [splits-1][NT/4 column quads][128 rows][4] fp32, so that the 32 rows of a warp
        // move 512 contiguous bytes per 16-byte access.
        float part[HC];
        float* red = reinterpret_cast<float*>(smem + (C::RED_OWN ? C::OFF_RED : 0));
        const int row = sub * 32 + lane;
        cluster_wait();  // every CTA of the cluster has initialised its barriers
        if (epi) {
            const bool ok = mbar_wait(&accf[0], 0, p.status, 58);
            if (!C::RED_OWN && split == 0 && warp == 2 + kWtDeqWarps && lane == 0)
                for (uint32_t sp = 1; sp < splits; ++sp) mbar_arrive_cluster(mapa_shared(smem_u32(rready), sp));
            tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + static_cast<uint32_t>(half * HC);
#pragma unroll
            for (int c = 0; c < HC; c += 16) {
                uint32_t rr[16];
                tmem_ld_32x32b_x16(t_row + c, rr);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) part[c + j] = ok ? __uint_as_float(rr[j]) : 0.0f;
            }
            tc_fence_before();
        }
        if (epi && split != 0 && (C::RED_OWN || mbar_wait_cluster(rready, 0, p.status, 59))) {
            const uint32_t dst =
                mapa_shared(smem_u32(red + (((split - 1) * (NT / 4) + half * HC / 4) * 128 + row) * 4), 0);
            const uint32_t bar = mapa_shared(smem_u32(rfull), 0);
#pragma unroll
            for (int v4 = 0; v4 < HC / 4; ++v4)
                st_async_v4(dst + v4 * 128 * 16, part[4 * v4], part[4 * v4 + 1], part[4 * v4 + 2], part[4 * v4 + 3],
                            bar);
        }
        if (epi && split == 0) {
            const int tt = first % p.t_tiles, wt = first / p.t_tiles;
            const bool got = mbar_wait(rfull, 0, p.status, 60);
            for (uint32_t sp = 1; got && sp < splits; ++sp) {
                const float4* src = reinterpret_cast<const float4*>(red) + ((sp - 1) * (NT / 4) + half * HC / 4) * 128 + row;
#pragma unroll
                for (int v4 = 0; v4 < HC / 4; ++v4) {
                    const float4 q = src[v4 * 128];
                    part[4 * v4] = __fadd_rn(part[4 * v4], q.x);
                    part[4 * v4 + 1] = __fadd_rn(part[4 * v4 + 1], q.y);
                    part[4 * v4 + 2] = __fadd_rn(part[4 * v4 + 2], q.z);
                    part[4 * v4 + 3] = __fadd_rn(part[4 * v4 + 3], q.w);
                }
            }
#pragma unroll
            for (int j = 0; j < HC; ++j) store(tt, wt, j, part[j]);
        }
        __syncthreads();
    }
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

// bf16 out [M][N]: boxes of 32 columns (64 bytes) x 32 rows, 64B swizzle (16-byte piece q of row r
// at piece q ^ ((r >> 1) & 3)); TMA stores clip at the M and N edges.
bool make_out32_map(CUtensorMap* m, void* out, int64_t M, int64_t N) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, out, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
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

// packed FP4 W [N][K/2]: boxes of 128 bytes (256 elements) x 128 rows, 128B swizzle.
bool make_w4_wide_map(CUtensorMap* m, const void* W, int64_t N, int64_t K) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    cuuint32_t box[2] = {128, 128};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(W), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Swizzled W scales as rows of 256 bytes; a box is `tiles` consecutive 512-byte tiles of a row group.
bool make_w_sf_tiles_map(CUtensorMap* m, const void* sf, int64_t rows, int64_t kblocks, uint32_t tiles) {
    auto enc = encode_fn();
    if (!enc) return false;
    const uint64_t half_rows = static_cast<uint64_t>(swizzled_sf_bytes(rows, kblocks) / 256);
    cuuint64_t dims[2] = {256, half_rows};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {256, 2 * tiles};
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
    CUtensorMap ta, tw, tsf, to;
    if (!make_a16_map(&ta, A, M, K, a_rows) || !make_w4_map(&tw, Wq, N, K, BN) ||
        !make_w_sf_map(&tsf, Wsf, N, K / C::BS))
        return MXQ_ERR_CUDA;
    const bool tma_store = !F32 && N % 8 == 0;
    if (!tma_store)
        to = tw;  // the output is stored directly; the map is not used
    else if (!make_out32_map(&to, out, M, N))
        return MXQ_ERR_CUDA;
    W16Args args = {};
    args.tma_store = tma_store ? 1 : 0;
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
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles < sm_count() ? tiles : sm_count()));
    cfg.blockDim = dim3(kW16Threads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, ta, tw, tsf, to, args) == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

template <int FMT, int NT, int STAGES, int AS, bool SPLIT, int DQW, bool F32>
int run_w16t(const void* A, const void* Wq, const uint8_t* Wsf, const float* g_w, int64_t M, int64_t N, int64_t K,
             void* out, cudaStream_t stream, int splits) {
    using C = W16TCfg<FMT, NT, STAGES, AS, SPLIT>;
    auto kern = w4a16_tmem_kernel<FMT, NT, STAGES, AS, SPLIT, DQW, F32>;
    const uint32_t act_rows = static_cast<uint32_t>(M >= NT ? NT : ceil_div(M, 8) * 8);
    CUtensorMap ta, tw, tsf;
    if (!make_a16_map(&ta, A, M, K, act_rows) || !make_w4_wide_map(&tw, Wq, N, K) ||
        !make_w_sf_tiles_map(&tsf, Wsf, N, K / C::BS, C::SF_ATOMS))
        return MXQ_ERR_CUDA;
    W16TArgs args = {};
    args.g_w = g_w;
    args.out = out;
    args.M = static_cast<int>(M);
    args.N = static_cast<int>(N);
    args.K = static_cast<int>(K);
    args.sf_col_tiles = static_cast<int>(ceil_div(K / C::BS, 4));
    args.t_tiles = static_cast<int>(ceil_div(M, NT));
    args.w_tiles = static_cast<int>(ceil_div(N, 128));
    args.k_stages = static_cast<int>(ceil_div(K, kWtK));
    args.k_split = static_cast<uint32_t>(splits);
    args.act_box_bytes = act_rows * 128;
    args.status = status_ptr();
    int dev = 0;
    cudaGetDevice(&dev);
    static bool attr_done[64] = {};
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
            return MXQ_ERR_CUDA;
        attr_done[dev] = true;
    }
    const int64_t tiles = static_cast<int64_t>(args.t_tiles) * args.w_tiles;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kWtThreads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    // programmatic serialization: the prologue may overlap the tail of the previous kernel
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if constexpr (SPLIT) {
        cfg.gridDim = dim3(static_cast<unsigned>(tiles * splits));
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = static_cast<unsigned>(splits);
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    } else {
        // 16 dequantizing warps include the epilogue warps: every CTA must own exactly one tile
        if (DQW == 16 && tiles > sm_count()) return MXQ_ERR_UNSUPPORTED;
        cfg.gridDim = dim3(static_cast<unsigned>(tiles < sm_count() ? tiles : sm_count()));
    }
    if (cudaLaunchKernelEx(&cfg, kern, ta, tw, tsf, args) != cudaSuccess) return MXQ_ERR_CUDA;
    return MXQ_OK;
}

// K splits for a few-tile problem: as many as keep every cluster resident at once (at most
// max_splits), each split owning at least 2 K stages of 256.
int w16_splits(int64_t tiles, int64_t k_stages, int max_splits) {
    int64_t s = sm_count() / (tiles > 0 ? tiles : 1);
    if (s > max_splits) s = max_splits;
    if (s > k_stages / 2) s = k_stages / 2;
    if (s < 2) return 1;
    // the kernel gives each split ceil(k_stages / s) stages: drop splits that would get none
    // (9 stages over 4 would leave the last one empty)
    const int64_t per = ceil_div(k_stages, s);
    return static_cast<int>(ceil_div(k_stages, per));
}

template <int FMT, bool F32>
int dispatch_w16(const void* A, const void* Wq, const uint8_t* Wsf, const float* g_w, int64_t M, int64_t N,
                 int64_t K, void* out, cudaStream_t stream) {
    // More than 128 tokens: dequantize each 256-row weight tile once into shared memory for two
    // M=128 MMAs (256 x 256 tiles).  Up to 128 tokens the weight stream dominates: weights go to
    // TMEM, 256 K per stage, split along K when there are few tiles.
    if (M > 128) return run_w16<FMT, 2, 256, F32>(A, Wq, Wsf, g_w, M, N, K, out, stream);
    const int64_t w_tiles = ceil_div(N, 128), k_stages = ceil_div(K, kWtK);
    // With one tile per CTA (a K split, or no more tiles than SMs) the epilogue warps have nothing
    // to overlap and dequantize too (16 warps); otherwise 8 warps dequantize while 8 drain.
    if (M > 32) {
        const int64_t tiles = w_tiles * ceil_div(M, 64);
        const int s = w16_splits(tiles, k_stages, 4);
        if (s > 1) return run_w16t<FMT, 64, 4, 3, true, 16, F32>(A, Wq, Wsf, g_w, M, N, K, out, stream, s);
        return tiles <= sm_count() ? run_w16t<FMT, 64, 4, 3, false, 16, F32>(A, Wq, Wsf, g_w, M, N, K, out, stream, 1)
                                   : run_w16t<FMT, 64, 4, 3, false, 8, F32>(A, Wq, Wsf, g_w, M, N, K, out, stream, 1);
    }
    const int s = w16_splits(w_tiles, k_stages, 4);
    if (s > 1) return run_w16t<FMT, 32, 5, 3, true, 16, F32>(A, Wq, Wsf, g_w, M, N, K, out, stream, s);
    return w_tiles <= sm_count() ? run_w16t<FMT, 32, 6, 3, false, 16, F32>(A, Wq, Wsf, g_w, M, N, K, out, stream, 1)
                                 : run_w16t<FMT, 32, 6, 3, false, 8, F32>(A, Wq, Wsf, g_w, M, N, K, out, stream, 1);
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
