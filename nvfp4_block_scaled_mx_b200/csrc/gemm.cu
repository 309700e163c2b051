// gemm.cu -- block-scaled GEMM on the sm_100a tensor cores (tcgen05), out = alpha * dq(A) dq(B)^T.
//
// Three kernels share the MMA, scale and epilogue plumbing, chosen on the host by shape:
//   gemm_pair_kernel    M > 128: two-CTA clusters computing 256 x BN tiles (cta_group::2);
//   gemm_splitk_kernel  M <= 128 with too few output tiles for the SMs: K split over a cluster,
//                       partials reduced through distributed shared memory;
//   gemm_kernel         M <= 128 otherwise, described here.
// Two more kernels serve the linear layer in one launch, quantizing its bf16 activations themselves:
//   gemm_decode_kernel  up to 32 tokens (weights as the 128-row MMA operand, tokens as N = 32);
//   gemm_rowq_kernel    more tokens and N <= 128 (each activation row read once, as bf16).
//
// gemm_kernel: one persistent CTA per SM, warp-specialised:
//   warp 0       TMA producer: A and B tiles (128-byte K slices, 128B-swizzled) and their
//                swizzled scale tiles (bulk copies) into a STAGES-deep shared-memory ring;
//   warp 1       TMEM owner and MMA issuer: 4 block-scaled MMAs per stage into an fp32
//                accumulator of 128 lanes x BN columns;
//   warps 2-9    epilogue: tcgen05.ld of the accumulator (two warps per 32-lane sub-partition, each
//                owning half of the BN columns), alpha scaling, bf16 RNE or fp32 conversion,
//                stores with M/N tail masking;
//   warps 10-13  scale staging: each writes the stage's scale tiles into its own TMEM
//                sub-partition with tcgen05.st (the layout tcgen05.cp .32x128b.warpx4 would produce).
//                Keeping the scale writes off the MMA thread keeps its tensor-core queue to MMAs
//                only; issuing tcgen05.cp from the MMA thread cost ~300 clk per stage on B200.
// Tiles are 128 x BN (BN = 256 or 128) and walked M-fastest so the CTAs resident at one time
// share the same few B tiles and all of A through L2.
//
// Formats (KIND): 0 MXFP4 kind::mxf4 (E2M1 x E2M1, UE8M0 per 32, K = 64 per MMA)
//                 1 NVFP4 kind::mxf4nvf4 (E2M1 x E2M1, UE4M3 per 16, K = 64 per MMA)
//                 2 MXFP8 kind::mxf8f6f4 (E4M3 x E4M3, UE8M0 per 32, K = 32 per MMA)
// Every stage holds 128 bytes of K per row (256 FP4 or 128 FP8 elements), i.e. 4 MMAs.
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "mxq_device.cuh"
#include "mxq_internal.h"
#include "quant_block.cuh"

namespace mxq {

// cuTensorMapEncodeTiled from the driver, looked up once.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

namespace {

constexpr int kBM = 128;
constexpr int kEpiWarps = 8;
constexpr int kSfWarps = 4;
constexpr int kThreads = (2 + kEpiWarps + kSfWarps) * 32;

template <int KIND>
struct Fmt;
template <>
struct Fmt<0> {
    static constexpr int BS = 32, EPB = 2, MMA_K = 64;
};
template <>
struct Fmt<1> {
    static constexpr int BS = 16, EPB = 2, MMA_K = 64;
};
template <>
struct Fmt<2> {
    static constexpr int BS = 32, EPB = 1, MMA_K = 32;
};

template <int KIND, int BN, int STAGES>
struct Cfg {
    static constexpr int BS = Fmt<KIND>::BS, EPB = Fmt<KIND>::EPB, MMA_K = Fmt<KIND>::MMA_K;
    static constexpr int BK = 128 * EPB;          // elements of K per stage
    static constexpr int KSTEPS = BK / MMA_K;     // MMAs per stage (4)
    static constexpr int KB_PER_MMA = MMA_K / BS; // scale blocks per MMA and row (2 / 4 / 1)
    static constexpr int SF_ATOMS = BK / BS / 4;  // 512-byte scale tiles per 128 rows per stage
    static constexpr int BGROUPS = BN / 128;
    static constexpr int A_BYTES = kBM * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int SFA_BYTES = SF_ATOMS * 512;
    static constexpr int SFB_BYTES = SF_ATOMS * BGROUPS * 512;
    static constexpr int ACC_STAGES = (BN == 256) ? 1 : 2;
    // TMEM columns: accumulators first, then one scale slot per pipeline stage.
    static constexpr int SF_COLS_A = SF_ATOMS * 4;
    static constexpr int SF_COLS_B = SF_ATOMS * (BN / 32);
    static constexpr int SF_COLS_STAGE = SF_COLS_A + SF_COLS_B;
    static constexpr int SF_TMEM_BASE = ACC_STAGES * BN;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(SF_TMEM_BASE + STAGES * SF_COLS_STAGE <= 512, "TMEM budget");
    static_assert(KSTEPS == 4, "4 MMAs per 128-byte stage");
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
    static constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_BYTES;
    static constexpr int N_BARS = 3 * STAGES + 2 * ACC_STAGES;
    static constexpr int OFF_SLOT = OFF_BAR + N_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_SLOT + 16 + 1024;  // + slack for 1024-byte alignment
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct GemmArgs {
    const uint8_t* a_sf;
    const uint8_t* b_sf;
    const float* g_a;
    const float* g_b;
    void* out;
    int M, N, K;
    int sf_col_tiles;  // ceil(K / bs / 4)
    int b_row_tiles;   // ceil(N / 128)
    int m_tiles, n_tiles, k_stages;
    int* status;
    uint32_t k_split;      // K-split kernels: CTAs per cluster sharing one output tile
    uint32_t a_box_bytes;  // split-K kernel: bytes of one A load (rows rounded up to 8, <= 128)
    uint32_t tma_store;    // pair kernel: bf16 output written through TMA stores (N % 8 == 0)
    const void* x;         // few-token and small-N kernels, which quantize their own A: the bf16 activations [M, K]
    int group_m;           // pair kernel: M tiles per raster group (m_tiles: plain M-fastest order)
};

// Pair-kernel tile order: groups of group_m M tiles, M-fastest inside a group, groups in M order.
// A wave of tiles then touches group_m A tiles and about (pairs / group_m) B tiles, instead of
// every A tile; group_m = m_tiles is the plain M-fastest walk.
__device__ __forceinline__ void pair_tile_coords(int tile, int m_tiles, int n_tiles, int group_m, int& mt, int& nt) {
    const int per_group = group_m * n_tiles;
    const int grp = tile / per_group;
    const int first = grp * group_m;
    const int gs = min(group_m, m_tiles - first);
    const int local = tile - grp * per_group;
    mt = first + local % gs;
    nt = local / gs;
}

template <int KIND, int BN, int STAGES, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                const GemmArgs p) {
    using C = Cfg<KIND, BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* sfready = empty + STAGES;
    uint64_t* accf = sfready + STAGES;
    uint64_t* acce = accf + C::ACC_STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_SLOT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tma_a);
        prefetch_tmap(&tma_b);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sfready[s], kSfWarps);
        }
        for (int a = 0; a < C::ACC_STAGES; ++a) {
            mbar_init(&accf[a], 1);
            mbar_init(&acce[a], kEpiWarps * 32);
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
    const uint32_t tmem_base = *tmem_slot;

    // operands may come from the kernel launched just before this one on the stream
    pdl_wait();
    pdl_launch_dependents();  // the next kernel on the stream may start its prologue

    const int num_tiles = p.m_tiles * p.n_tiles;
    auto groups_of = [&](int tile) {
        const int nt = tile / p.m_tiles;
        int groups = 0;
#pragma unroll
        for (int g = 0; g < C::BGROUPS; ++g) groups += (nt * C::BGROUPS + g < p.b_row_tiles) ? 1 : 0;
        return groups;
    };

    if (warp == 0) {
        // TMA producer: the whole warp runs the loop; one elected lane issues
        const uint64_t pol_a = policy_evict_last();
        const uint64_t pol_b = policy_evict_normal();
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
            const int groups = groups_of(tile);
            for (int ks = 0; ks < p.k_stages; ++ks) {
                if (!mbar_wait_warp(&empty[stage], phase ^ 1u, p.status, 1)) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    const int atoms = min(C::SF_ATOMS, p.sf_col_tiles - ks * C::SF_ATOMS);
                    const uint32_t bytes = C::A_BYTES + C::B_BYTES + atoms * 512 * (1 + groups);
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    tma_load_2d(&tma_a, &full[stage], smem + C::OFF_A + stage * C::A_BYTES, ks * 128, mt * kBM, pol_a);
                    tma_load_2d(&tma_b, &full[stage], smem + C::OFF_B + stage * C::B_BYTES, ks * 128, nt * BN, pol_b);
                    const int64_t kcol = static_cast<int64_t>(ks) * C::SF_ATOMS;
                    bulk_load(smem + C::OFF_SFA + stage * C::SFA_BYTES,
                              p.a_sf + (static_cast<int64_t>(mt) * p.sf_col_tiles + kcol) * 512, atoms * 512,
                              &full[stage]);
                    for (int g = 0; g < groups; ++g)
                        bulk_load(smem + C::OFF_SFB + stage * C::SFB_BYTES + g * C::SF_ATOMS * 512,
                                  p.b_sf + (static_cast<int64_t>(nt * C::BGROUPS + g) * p.sf_col_tiles + kcol) * 512,
                                  atoms * 512, &full[stage]);
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        // MMA issuer: the whole warp runs the loop; one elected lane issues
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            if (!mbar_wait_warp(&acce[acc], acc_phase ^ 1u, p.status, 2)) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
            for (int ks = 0; ks < p.k_stages; ++ks) {
                // operands landed (TMA) and the stage's scales sit in its TMEM slot (staging warps)
                if (!mbar_wait_warp(&full[stage], phase, p.status, 3) || !mbar_wait_warp(&sfready[stage], phase, p.status, 5)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sf_col = tmem_base + C::SF_TMEM_BASE + stage * C::SF_COLS_STAGE;
                const uint32_t a_s = smem_u32(smem + C::OFF_A + stage * C::A_BYTES);
                const uint32_t b_s = smem_u32(smem + C::OFF_B + stage * C::B_BYTES);
                if (elect_one()) {
#pragma unroll
                    for (int j = 0; j < C::KSTEPS; ++j) {
                        if (ks * C::BK + j * C::MMA_K < p.K) {
                            const int kb = j * C::KB_PER_MMA;  // first scale block of this MMA in the stage
                            const int atom = kb >> 2;
                            const uint32_t idesc = mma_idesc<KIND>(kBM, BN, static_cast<uint32_t>(kb & 3));
                            mma_block_scaled<KIND>(d_tmem, smem_desc(a_s + j * 32, 16, 1024, kLayoutSwizzle128B),
                                                   smem_desc(b_s + j * 32, 16, 1024, kLayoutSwizzle128B), idesc,
                                                   sf_col + atom * 4, sf_col + C::SF_COLS_A + atom * (BN / 32),
                                                   (ks | j) != 0 ? 1u : 0u);
                        }
                    }
                    tc_commit(&empty[stage]);
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (elect_one()) tc_commit(&accf[acc]);
            __syncwarp();
            if (++acc == C::ACC_STAGES) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    } else if (warp >= 2 + kEpiWarps) {
        // scale staging: lane l of every staging warp holds row l of each 512-byte scale tile
        // (16 bytes = 4 TMEM columns) and writes it into its own sub-partition, so all four
        // sub-partitions see the same replicated tile.
        const int sub = warp & 3;
        const uint32_t lane_addr = static_cast<uint32_t>(sub * 32) << 16;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            for (int ks = 0; ks < p.k_stages; ++ks) {
                if (!mbar_wait(&full[stage], phase, p.status, 6)) {
                    ok = false;
                    break;
                }
                uint32_t r[C::SF_COLS_STAGE];
                const uint32_t sfa_s = smem_u32(smem + C::OFF_SFA + stage * C::SFA_BYTES) + lane * 16;
                const uint32_t sfb_s = smem_u32(smem + C::OFF_SFB + stage * C::SFB_BYTES) + lane * 16;
#pragma unroll
                for (int a = 0; a < C::SF_ATOMS; ++a) {
                    const uint4 v = ld_shared_v4(sfa_s + a * 512);
                    r[a * 4 + 0] = v.x;
                    r[a * 4 + 1] = v.y;
                    r[a * 4 + 2] = v.z;
                    r[a * 4 + 3] = v.w;
                }
#pragma unroll
                for (int a = 0; a < C::SF_ATOMS; ++a) {
#pragma unroll
                    for (int g = 0; g < C::BGROUPS; ++g) {
                        const uint4 v = ld_shared_v4(sfb_s + (g * C::SF_ATOMS + a) * 512);
                        const int c = C::SF_COLS_A + a * (BN / 32) + g * 4;
                        r[c + 0] = v.x;
                        r[c + 1] = v.y;
                        r[c + 2] = v.z;
                        r[c + 3] = v.w;
                    }
                }
                tmem_st_cols<C::SF_COLS_STAGE>(tmem_base + lane_addr + C::SF_TMEM_BASE + stage * C::SF_COLS_STAGE, r);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfready[stage]);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        constexpr int COLS = BN / 2;  // accumulator columns owned by this warp
        const int sub = warp & 3;     // TMEM sub-partition this warp may read
        const int col0 = ((warp - 2) >> 2) * COLS;
        const int row = sub * 32 + lane;
        const float alpha = (KIND == 1) ? __fmul_rn(*p.g_a, *p.g_b) : 1.0f;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int mt = tile % p.m_tiles, nt = tile / p.m_tiles;
            if (!mbar_wait(&accf[acc], acc_phase, p.status, 4)) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) +
                                   static_cast<uint32_t>(acc * BN + col0);
            const int m = mt * kBM + row;
            const int n0 = nt * BN + col0;
            if constexpr (!OUT_F32) {
                __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(m) * p.N;
                const bool vec = (n0 + COLS <= p.N) && (p.N & 7) == 0;
                // drain this warp's columns 64 at a time into registers (two TMEM loads per wait)
                // and store them; the accumulator is released once its last columns are loaded, so
                // the last stores overlap the next tile's mainloop
#pragma unroll
                for (int hb = 0; hb < COLS; hb += 64) {
                    uint32_t packed[32];
                    {
                        uint32_t r0[32], r1[32];
                        tmem_ld_32x32b_x32(t_row + hb, r0);
                        tmem_ld_32x32b_x32(t_row + hb + 32, r1);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float lo = __uint_as_float(r0[2 * i]), hi = __uint_as_float(r0[2 * i + 1]);
                            float lo1 = __uint_as_float(r1[2 * i]), hi1 = __uint_as_float(r1[2 * i + 1]);
                            if (KIND == 1) {
                                lo = __fmul_rn(lo, alpha);
                                hi = __fmul_rn(hi, alpha);
                                lo1 = __fmul_rn(lo1, alpha);
                                hi1 = __fmul_rn(hi1, alpha);
                            }
                            const __nv_bfloat162 b0 = __floats2bfloat162_rn(lo, hi);
                            const __nv_bfloat162 b1 = __floats2bfloat162_rn(lo1, hi1);
                            packed[i] = *reinterpret_cast<const uint32_t*>(&b0);
                            packed[16 + i] = *reinterpret_cast<const uint32_t*>(&b1);
                        }
                    }
                    if (hb + 64 == COLS) {
                        tc_fence_before();
                        mbar_arrive(&acce[acc]);
                    }
                    if (m < p.M) {
                        if (vec) {
                            uint4* dst = reinterpret_cast<uint4*>(orow + n0 + hb);
#pragma unroll
                            for (int v = 0; v < 8; ++v)
                                dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
                        } else {
                            uint16_t* o16 = reinterpret_cast<uint16_t*>(orow);
#pragma unroll
                            for (int v = 0; v < 32; ++v) {
                                const int n = n0 + hb + 2 * v;
                                if (n < p.N) o16[n] = static_cast<uint16_t>(packed[v] & 0xFFFFu);
                                if (n + 1 < p.N) o16[n + 1] = static_cast<uint16_t>(packed[v] >> 16);
                            }
                        }
                    }
                }
            } else {
                float* orow = static_cast<float*>(p.out) + static_cast<int64_t>(m) * p.N;
                const bool vec = (p.N & 3) == 0;
#pragma unroll 1
                for (int c = 0; c < COLS / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(t_row + c * 32, r);
                    tmem_ld_wait();
                    if (m < p.M) {
                        const int nb = n0 + c * 32;
                        if (vec && nb + 32 <= p.N) {
                            float4* dst = reinterpret_cast<float4*>(orow + nb);
#pragma unroll
                            for (int v = 0; v < 8; ++v) {
                                float4 f;
                                f.x = __fmul_rn(__uint_as_float(r[4 * v]), alpha);
                                f.y = __fmul_rn(__uint_as_float(r[4 * v + 1]), alpha);
                                f.z = __fmul_rn(__uint_as_float(r[4 * v + 2]), alpha);
                                f.w = __fmul_rn(__uint_as_float(r[4 * v + 3]), alpha);
                                dst[v] = f;
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (nb + i < p.N) orow[nb + i] = __fmul_rn(__uint_as_float(r[i]), alpha);
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(&acce[acc]);
            }
            if (++acc == C::ACC_STAGES) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ split-K kernel (M <= 128)
//
// Few-token problems (decode) have too few 128 x 128 output tiles to keep every SM streaming
// weights.  Here a cluster of S CTAs shares one output tile, each CTA accumulating a contiguous
// share of the K stages; the S partial accumulators are reduced through distributed shared memory
// in the leader (rank 0) CTA, which alone writes the output.  No global workspace is used.
// Roles are those of gemm_kernel (warp 0 TMA, warp 1 MMA, warps 2-9 epilogue, 10-13 scale staging).

constexpr uint32_t kMaxSplits = 4;

template <int KIND, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_splitk_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                       const GemmArgs p) {
    constexpr int BN = 128, STAGES = 6;
    using C = Cfg<KIND, BN, STAGES>;
    static_assert((kMaxSplits - 1) * 128 * BN * 4 <= STAGES * (C::A_BYTES + C::B_BYTES), "reduction buffer");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* sfready = empty + STAGES;
    uint64_t* accf = sfready + STAGES;
    uint64_t* rready = accf + 1;  // non-leaders: the leader's operand ring is free for the partials
    uint64_t* rfull = accf + 2;   // leader: every partial has landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_SLOT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t split = cluster_ctarank();
    const uint32_t splits = p.k_split;
    const int nt = static_cast<int>(blockIdx.x / splits);
    const int per = (p.k_stages + static_cast<int>(splits) - 1) / static_cast<int>(splits);
    const int k0 = static_cast<int>(split) * per;
    const int k1 = min(p.k_stages, k0 + per);
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tma_a);
        prefetch_tmap(&tma_b);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sfready[s], kSfWarps);
        }
        mbar_init(accf, 1);
        mbar_init(rready, 1);
        mbar_init(rfull, 1);
        // the partials of rows < M from the other splits-1 CTAs, counted in bytes
        if (split == 0) mbar_arrive_expect_tx(rfull, (splits - 1) * static_cast<uint32_t>(min(p.M, 128)) * BN * 4);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_arrive_relaxed();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();
    pdl_launch_dependents();  // the next kernel on the stream may start its prologue

    const bool b_group = nt < p.b_row_tiles;  // always true: one 128-row B group per tile
    if (warp == 0) {
        // TMA producer: the whole warp runs the loop; one elected lane issues
        const uint64_t pol = policy_evict_first();
        int stage = 0;
        uint32_t phase = 0;
        for (int ks = k0; ks < k1; ++ks) {
            if (!mbar_wait_warp(&empty[stage], phase ^ 1u, p.status, 21)) break;
            if (elect_one()) {
                const int atoms = min(C::SF_ATOMS, p.sf_col_tiles - ks * C::SF_ATOMS);
                // A rows past M are not loaded: they only feed accumulator rows that are never stored
                mbar_arrive_expect_tx(&full[stage], p.a_box_bytes + C::B_BYTES + atoms * 512 * (1 + (b_group ? 1 : 0)));
                tma_load_2d(&tma_a, &full[stage], smem + C::OFF_A + stage * C::A_BYTES, ks * 128, 0, pol);
                tma_load_2d(&tma_b, &full[stage], smem + C::OFF_B + stage * C::B_BYTES, ks * 128, nt * BN, pol);
                const int64_t kcol = static_cast<int64_t>(ks) * C::SF_ATOMS;
                bulk_load(smem + C::OFF_SFA + stage * C::SFA_BYTES, p.a_sf + kcol * 512, atoms * 512, &full[stage]);
                if (b_group)
                    bulk_load(smem + C::OFF_SFB + stage * C::SFB_BYTES,
                              p.b_sf + (static_cast<int64_t>(nt) * p.sf_col_tiles + kcol) * 512, atoms * 512,
                              &full[stage]);
            }
            __syncwarp();
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
    } else if (warp == 1) {
        // MMA issuer: the whole warp runs the loop; one elected lane issues
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int ks = k0; ks < k1; ++ks) {
            if (!mbar_wait_warp(&full[stage], phase, p.status, 23) || !mbar_wait_warp(&sfready[stage], phase, p.status, 25)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t sf_col = tmem_base + C::SF_TMEM_BASE + stage * C::SF_COLS_STAGE;
            const uint32_t a_s = smem_u32(smem + C::OFF_A + stage * C::A_BYTES);
            const uint32_t b_s = smem_u32(smem + C::OFF_B + stage * C::B_BYTES);
            if (elect_one()) {
#pragma unroll
                for (int j = 0; j < C::KSTEPS; ++j) {
                    if (ks * C::BK + j * C::MMA_K < p.K) {
                        const int kb = j * C::KB_PER_MMA;
                        const int atom = kb >> 2;
                        mma_block_scaled<KIND>(tmem_base, smem_desc(a_s + j * 32, 16, 1024, kLayoutSwizzle128B),
                                               smem_desc(b_s + j * 32, 16, 1024, kLayoutSwizzle128B),
                                               mma_idesc<KIND>(kBM, BN, static_cast<uint32_t>(kb & 3)),
                                               sf_col + atom * 4, sf_col + C::SF_COLS_A + atom * (BN / 32),
                                               (ks > k0 || j > 0) ? 1u : 0u);
                    }
                }
                tc_commit(&empty[stage]);
            }
            __syncwarp();
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (ok && elect_one()) tc_commit(accf);
        __syncwarp();
    } else if (warp >= 2 + kEpiWarps) {
        // scale staging (warps 10-13, one per TMEM sub-partition)
        const int sub = warp & 3;
        const uint32_t lane_addr = static_cast<uint32_t>(sub * 32) << 16;
        int stage = 0;
        uint32_t phase = 0;
        for (int ks = k0; ks < k1; ++ks) {
            if (!mbar_wait(&full[stage], phase, p.status, 26)) break;
            uint32_t r[C::SF_COLS_STAGE];

            const uint32_t sfa_s = smem_u32(smem + C::OFF_SFA + stage * C::SFA_BYTES) + lane * 16;
            const uint32_t sfb_s = smem_u32(smem + C::OFF_SFB + stage * C::SFB_BYTES) + lane * 16;
#pragma unroll
            for (int a = 0; a < C::SF_ATOMS; ++a) {
                const uint4 va = ld_shared_v4(sfa_s + a * 512);
                r[a * 4 + 0] = va.x;
                r[a * 4 + 1] = va.y;
                r[a * 4 + 2] = va.z;
                r[a * 4 + 3] = va.w;
                const uint4 vb = ld_shared_v4(sfb_s + a * 512);
                r[C::SF_COLS_A + a * 4 + 0] = vb.x;
                r[C::SF_COLS_A + a * 4 + 1] = vb.y;
                r[C::SF_COLS_A + a * 4 + 2] = vb.z;
                r[C::SF_COLS_A + a * 4 + 3] = vb.w;
            }
            tmem_st_cols<C::SF_COLS_STAGE>(tmem_base + lane_addr + C::SF_TMEM_BASE + stage * C::SF_COLS_STAGE, r);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sfready[stage]);
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
    }

    // reduction: every CTA's epilogue warps take their share of the partial tile into registers.
    // The leader frees its operand ring for the partials once its MMAs are done (a remote arrive
    // per other CTA); the others send their rows < M with st.async, counted in bytes on the
    // leader's barrier, and leave.  Layout in the leader: [splits-1][BN/4 column quads][128 rows][4]
    // fp32, so that the 32 rows of a warp move 512 contiguous bytes per 16-byte access.
    constexpr int COLS = BN / 2;
    const bool epi = warp >= 2 && warp < 2 + kEpiWarps;
    const int sub = warp & 3;
    const int col0 = ((warp - 2) >> 2) * COLS;
    const int row = sub * 32 + lane;
    float* red = reinterpret_cast<float*>(smem);
    float acc[COLS];
    cluster_wait();  // every CTA of the cluster has initialised its barriers
    if (epi) {
        const bool ok = mbar_wait(accf, 0, p.status, 24);
        if (split == 0 && warp == 2 && lane == 0)
            for (uint32_t sp = 1; sp < splits; ++sp) mbar_arrive_cluster(mapa_shared(smem_u32(rready), sp));
        tc_fence_after();
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + static_cast<uint32_t>(col0);
#pragma unroll
        for (int c = 0; c < COLS / 32; ++c) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_row + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[c * 32 + i] = ok ? __uint_as_float(r[i]) : 0.0f;
        }
        tc_fence_before();
    }
    if (epi && split != 0 && row < p.M && mbar_wait_cluster(rready, 0, p.status, 27)) {
        const uint32_t dst = mapa_shared(smem_u32(red + (((split - 1) * (BN / 4) + col0 / 4) * 128 + row) * 4), 0);
        const uint32_t bar = mapa_shared(smem_u32(rfull), 0);
#pragma unroll
        for (int v = 0; v < COLS / 4; ++v)
            st_async_v4(dst + v * 128 * 16, acc[4 * v], acc[4 * v + 1], acc[4 * v + 2], acc[4 * v + 3], bar);
    }
    if (epi && split == 0 && row < p.M) {
        const bool got = mbar_wait(rfull, 0, p.status, 28);
        for (uint32_t sp = 1; got && sp < splits; ++sp) {
            const float4* src = reinterpret_cast<const float4*>(red) + ((sp - 1) * (BN / 4) + col0 / 4) * 128 + row;
#pragma unroll
            for (int v = 0; v < COLS / 4; ++v) {
                const float4 q = src[v * 128];
                acc[4 * v] = __fadd_rn(acc[4 * v], q.x);
                acc[4 * v + 1] = __fadd_rn(acc[4 * v + 1], q.y);
                acc[4 * v + 2] = __fadd_rn(acc[4 * v + 2], q.z);
                acc[4 * v + 3] = __fadd_rn(acc[4 * v + 3], q.w);
            }
        }
        const float alpha = (KIND == 1) ? __fmul_rn(*p.g_a, *p.g_b) : 1.0f;
        const int n0 = nt * BN + col0;
        if constexpr (!OUT_F32) {
            __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(row) * p.N;
            uint32_t packed[COLS / 2];
#pragma unroll
            for (int i = 0; i < COLS / 2; ++i) {
                const float lo = KIND == 1 ? __fmul_rn(acc[2 * i], alpha) : acc[2 * i];
                const float hi = KIND == 1 ? __fmul_rn(acc[2 * i + 1], alpha) : acc[2 * i + 1];
                const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
                packed[i] = *reinterpret_cast<const uint32_t*>(&b);
            }
            if (n0 + COLS <= p.N && (p.N & 7) == 0) {
                uint4* dst = reinterpret_cast<uint4*>(orow + n0);
#pragma unroll
                for (int v = 0; v < COLS / 8; ++v)
                    dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
            } else {
                uint16_t* o16 = reinterpret_cast<uint16_t*>(orow);
#pragma unroll
                for (int v = 0; v < COLS / 2; ++v) {
                    const int n = n0 + 2 * v;
                    if (n < p.N) o16[n] = static_cast<uint16_t>(packed[v] & 0xFFFFu);
                    if (n + 1 < p.N) o16[n + 1] = static_cast<uint16_t>(packed[v] >> 16);
                }
            }
        } else {
            float* orow = static_cast<float*>(p.out) + static_cast<int64_t>(row) * p.N;
#pragma unroll
            for (int i = 0; i < COLS; ++i)
                if (n0 + i < p.N) orow[n0 + i] = __fmul_rn(acc[i], alpha);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ few-token linear kernel
//
// The decode-shaped linear layer (up to 32 tokens): streaming the weights is the whole cost, so a
// CTA owns 128 weight rows and a contiguous share of the K stages (the S CTAs of a cluster split K
// and reduce through distributed shared memory), and everything else hides under the weight
// stream.  The weights are the MMA's 128-row A operand and the tokens its N = 32 columns, so the
// accumulator is 32 TMEM columns whose 128 lanes span all four sub-partitions.  The bf16 tokens are
// quantized inside the kernel, in a ring of their own that runs ahead of the weight ring: the
// quantization of the first stages overlaps the latency of the first weight loads instead of
// following their arrival.
//   warp 0       TMA producer of the weight ring (codes, 128 rows x 128 bytes; their scale tiles)
//   warp 1       TMEM owner; copies each stage's weight and token scale tiles into TMEM
//                (tcgen05.cp) and issues the MMAs
//   warp 2       TMA producer of the bf16 token ring (boxes of 64 elements x 32 rows, 128B swizzle)
//   warps 3-10   quantize the token stages into the token-code ring (B operand layout) with the
//                streaming quantizer's arithmetic; then the epilogue.  Partials of the non-leader
//                CTAs go to a buffer of their own in the leader as soon as they are ready.
// WG = 2 (many weight rows, no K split): a CTA owns 256 weight rows as two 128-row MMA groups with an
// accumulator each, so that the tiles fit one wave and the tokens are quantized once per 256 rows.
template <int KIND, int WG>
struct DecCfg {
    static constexpr int BS = Fmt<KIND>::BS, EPB = Fmt<KIND>::EPB, MMA_K = Fmt<KIND>::MMA_K;
    static constexpr int BK = 128 * EPB;
    static constexpr int KSTEPS = BK / MMA_K;
    static constexpr int KB_PER_MMA = MMA_K / BS;
    static constexpr int SF_ATOMS = BK / BS / 4;
    static constexpr int TOK = 32;                   // MMA N: token rows (rows >= M are zero)
    // 4 to 7 weight stages measured the same (graph replays with the weights streamed from HBM)
    static constexpr int WSTAGES = (WG == 1) ? 5 : 4, XSTAGES = 2, TSTAGES = 5;
    static constexpr int W_BYTES = WG * 128 * 128;
    static constexpr int SF_BYTES = SF_ATOMS * 512;   // one 128-row scale tile column per stage
    static constexpr int SFW_BYTES = WG * SF_BYTES;   // the weight groups' scale tiles
    static constexpr int X_BOXES = BK / 64;
    static constexpr int X_BYTES = X_BOXES * TOK * 128;
    static constexpr int T_BYTES = TOK * 128;
    static constexpr int QWARPS = 8;
    static constexpr int THREADS = (3 + QWARPS) * 32;
    static constexpr int RED_BYTES = (WG == 1) ? (kMaxSplits - 1) * 128 * TOK * 4 : 0;  // WG = 2: no K split
    static constexpr int OFF_W = 0;
    static constexpr int OFF_X = OFF_W + WSTAGES * W_BYTES;
    static constexpr int OFF_T = OFF_X + XSTAGES * X_BYTES;
    static constexpr int OFF_RED = OFF_T + TSTAGES * T_BYTES;
    static constexpr int OFF_SFW = OFF_RED + RED_BYTES;
    static constexpr int OFF_SFT = OFF_SFW + WSTAGES * SFW_BYTES;
    static constexpr int OFF_TAB = OFF_SFT + TSTAGES * SF_BYTES;
    static constexpr int OFF_BAR = OFF_TAB + 1024;
    static constexpr int N_BARS = 2 * (WSTAGES + XSTAGES + TSTAGES) + 2;  // + accf, rfull
    static constexpr int OFF_SLOT = OFF_BAR + N_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_SLOT + 16 + 1024;
    static constexpr int SLOT_COLS = (WG + 1) * SF_ATOMS * 4;  // per weight stage: weight then token scale tiles
    static constexpr int SF_TMEM_BASE = WG * 32;                // one 32-column accumulator per weight group
    static constexpr uint32_t TMEM_COLS = 256;
    static_assert(KSTEPS == 4, "4 MMAs per stage");
    static_assert(SF_TMEM_BASE + WSTAGES * SLOT_COLS <= static_cast<int>(TMEM_COLS), "TMEM budget");
    static_assert(OFF_W % 1024 == 0 && OFF_X % 1024 == 0 && OFF_T % 1024 == 0, "swizzled buffers 1024-aligned");
    static_assert(WG * TOK * 128 * 2 <= XSTAGES * X_BYTES, "output staging tiles inside the token ring");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <int KIND, int WG, bool OUT_F32, int QRULE>
__global__ void __launch_bounds__(DecCfg<KIND, WG>::THREADS, 1)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tma_x, const __grid_constant__ CUtensorMap tma_w,
                       const __grid_constant__ CUtensorMap tma_out, const GemmArgs p) {
    using C = DecCfg<KIND, WG>;
    constexpr int WS = C::WSTAGES, XS = C::XSTAGES, TS = C::TSTAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* wempty = wfull + WS;
    uint64_t* xfull = wempty + WS;
    uint64_t* xempty = xfull + XS;
    uint64_t* tready = xempty + XS;
    uint64_t* tempty = tready + TS;
    uint64_t* accf = tempty + TS;
    uint64_t* rfull = accf + 1;  // leader: every partial has landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_SLOT);
    float* tab_d = reinterpret_cast<float*>(smem + C::OFF_TAB);
    float* tab_r = tab_d + 128;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t split = cluster_ctarank();
    const uint32_t splits = p.k_split;
    const int nt = static_cast<int>(blockIdx.x / splits);
    const int per = (p.k_stages + static_cast<int>(splits) - 1) / static_cast<int>(splits);
    const int k0 = static_cast<int>(split) * per;
    const int k1 = min(p.k_stages, k0 + per);
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tma_x);
        prefetch_tmap(&tma_w);
        for (int s = 0; s < WS; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&wempty[s], 1);
        }
        for (int s = 0; s < XS; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&xempty[s], C::QWARPS);
        }
        for (int s = 0; s < TS; ++s) {
            mbar_init(&tready[s], C::QWARPS);
            mbar_init(&tempty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(rfull, 1);
        // the other splits - 1 CTAs' partials (128 weight rows x 32 tokens, fp32), counted in bytes
        if (split == 0) mbar_arrive_expect_tx(rfull, (splits - 1) * 128u * C::TOK * 4u);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_arrive_relaxed();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();
    pdl_launch_dependents();  // the next kernel on the stream may start its prologue

    if (warp == 0) {
        // weight producer: the whole warp runs the loop; one elected lane issues
        const uint64_t pol = policy_evict_first();
        int stage = 0;
        uint32_t phase = 0;
        for (int ks = k0; ks < k1; ++ks) {
            if (!mbar_wait_warp(&wempty[stage], phase ^ 1u, p.status, 51)) break;
            if (elect_one()) {
                const int atoms = min(C::SF_ATOMS, p.sf_col_tiles - ks * C::SF_ATOMS);
                // row groups past N (WG = 2, last tile) load nothing: their rows are TMA zero fill
                const int groups = min(WG, p.b_row_tiles - nt * WG);
                mbar_arrive_expect_tx(&wfull[stage], C::W_BYTES + groups * atoms * 512);
                tma_load_2d(&tma_w, &wfull[stage], smem + C::OFF_W + stage * C::W_BYTES, ks * 128, nt * 128 * WG, pol);
                for (int g = 0; g < groups; ++g)
                    bulk_load(smem + C::OFF_SFW + stage * C::SFW_BYTES + g * C::SF_BYTES,
                              p.b_sf + (static_cast<int64_t>(nt * WG + g) * p.sf_col_tiles +
                                        static_cast<int64_t>(ks) * C::SF_ATOMS) * 512,
                              atoms * 512, &wfull[stage]);
            }
            __syncwarp();
            if (++stage == WS) {
                stage = 0;
                phase ^= 1u;
            }
        }
    } else if (warp == 1) {
        // scale copies and MMAs: the whole warp runs the loop; one elected lane issues
        int ws = 0, ts = 0;
        uint32_t wph = 0, tph = 0;
        bool ok = true;
        for (int ks = k0; ks < k1; ++ks) {
            if (!mbar_wait_warp(&wfull[ws], wph, p.status, 52) || !mbar_wait_warp(&tready[ts], tph, p.status, 53)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // TMEM scale slot of this weight stage (free: its previous MMAs completed before the
            // producer could refill the stage)
            // slot layout: the weight groups' scale tiles [g][atom], then the token scale tiles [atom]
            const uint32_t slot = tmem_base + C::SF_TMEM_BASE + ws * C::SLOT_COLS;
            const uint32_t sfw_s = smem_u32(smem + C::OFF_SFW + ws * C::SFW_BYTES);
            const uint32_t sft_s = smem_u32(smem + C::OFF_SFT + ts * C::SF_BYTES);
            const uint32_t w_s = smem_u32(smem + C::OFF_W + ws * C::W_BYTES);
            const uint32_t t_s = smem_u32(smem + C::OFF_T + ts * C::T_BYTES);
            constexpr int SFT_COL = WG * C::SF_ATOMS * 4;
            if (elect_one()) {
#pragma unroll
                for (int a = 0; a < C::SF_ATOMS; ++a) {
#pragma unroll
                    for (int g = 0; g < WG; ++g)
                        tc_cp_scales(slot + (g * C::SF_ATOMS + a) * 4,
                                     smem_desc(sfw_s + (g * C::SF_ATOMS + a) * 512, 0, 128, kLayoutNone));
                    tc_cp_scales(slot + SFT_COL + a * 4, smem_desc(sft_s + a * 512, 0, 128, kLayoutNone));
                }
#pragma unroll
                for (int j = 0; j < C::KSTEPS; ++j) {
                    if (ks * C::BK + j * C::MMA_K < p.K) {
                        const int kb = j * C::KB_PER_MMA;
                        const int atom = kb >> 2;
#pragma unroll
                        for (int g = 0; g < WG; ++g)
                            mma_block_scaled<KIND>(tmem_base + static_cast<uint32_t>(g * C::TOK),
                                                   smem_desc(w_s + g * 128 * 128 + j * 32, 16, 1024, kLayoutSwizzle128B),
                                                   smem_desc(t_s + j * 32, 16, 1024, kLayoutSwizzle128B),
                                                   mma_idesc<KIND>(128, C::TOK, static_cast<uint32_t>(kb & 3)),
                                                   slot + (g * C::SF_ATOMS + atom) * 4, slot + SFT_COL + atom * 4,
                                                   (ks > k0 || j > 0) ? 1u : 0u);
                    }
                }
                tc_commit(&wempty[ws]);
                tc_commit(&tempty[ts]);
            }
            __syncwarp();
            if (++ws == WS) {
                ws = 0;
                wph ^= 1u;
            }
            if (++ts == TS) {
                ts = 0;
                tph ^= 1u;
            }
        }
        if (ok && elect_one()) tc_commit(accf);
        __syncwarp();
    } else if (warp == 2) {
        // token producer: the stage's bf16 rows, boxes of 64 elements (128 bytes) x 32 rows
        const uint64_t pol = policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        for (int ks = k0; ks < k1; ++ks) {
            if (!mbar_wait_warp(&xempty[stage], phase ^ 1u, p.status, 54)) break;
            if (elect_one()) {
                mbar_arrive_expect_tx(&xfull[stage], C::X_BYTES);
#pragma unroll
                for (int b = 0; b < C::X_BOXES; ++b)
                    tma_load_2d(&tma_x, &xfull[stage], smem + C::OFF_X + stage * C::X_BYTES + b * C::TOK * 128,
                                (ks * C::BK + b * 64) * 2, 0, pol);
            }
            __syncwarp();
            if (++stage == XS) {
                stage = 0;
                phase ^= 1u;
            }
        }
    } else {
        // token quantizers: unit (row, j) = 32 elements; a warp takes the 32 token rows of one unit
        // column, so its 16-byte reads of the swizzled rows fall in distinct banks
        const int qt = (warp - 3) * 32 + lane;
        constexpr int UPR = C::BK / 32;  // units per token row and stage (8 FP4, 4 MXFP8)
        const bool active = qt < C::TOK * UPR;
        const int row = qt & 31, j = qt >> 5;
        float g_a = 1.0f;
        if constexpr (KIND == 1) {
            g_a = *p.g_a;
            if (qt < 128) {
                const float d = __fmul_rn(e4m3_decode_pos(static_cast<uint32_t>(qt)), g_a);
                tab_d[qt] = d;
                tab_r[qt] = __frcp_rn(d);  // fl(1/d), +inf for d = 0
            }
            named_barrier_sync(1, 32 * C::QWARPS);
        }
        int xs = 0, ts = 0;
        uint32_t xph = 0, tph = 0;
        for (int ks = k0; ks < k1; ++ks) {
            if (!mbar_wait_warp(&xfull[xs], xph, p.status, 55) || !mbar_wait_warp(&tempty[ts], tph ^ 1u, p.status, 56))
                break;
            if (active && static_cast<int64_t>(ks) * C::BK + j * 32 < p.K) {
                const uint32_t x_s = smem_u32(smem + C::OFF_X + xs * C::X_BYTES);
                const uint32_t t_s = smem_u32(smem + C::OFF_T + ts * C::T_BYTES);
                uint8_t* sft = smem + C::OFF_SFT + ts * C::SF_BYTES;
                uint32_t w[16];
                const uint32_t rb = x_s + (j >> 1) * C::TOK * 128 + row * 128;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 t = ld_shared_v4(rb + ((((j & 1) * 4 + i) ^ (row & 7)) << 4));
                    w[4 * i] = t.x;
                    w[4 * i + 1] = t.y;
                    w[4 * i + 2] = t.z;
                    w[4 * i + 3] = t.w;
                }
                uint32_t codes[8], seen = 0;
                const uint32_t sc = quantize32<KIND, (QRULE < 0 ? 0 : QRULE), false>(w, g_a, tab_d, tab_r, codes, seen);
                const uint32_t sw = static_cast<uint32_t>(row & 7);
                const uint32_t t_row = t_s + row * 128;
                // token scale atoms: the 32 token rows are rows 0-31 of a 128-row tile, byte row * 16 + block
                if constexpr (KIND == 2) {  // MXFP8: 32 bytes of codes, one scale block
                    st_shared_v4(t_row + (((2 * j) ^ sw) << 4), make_uint4(codes[0], codes[1], codes[2], codes[3]));
                    st_shared_v4(t_row + (((2 * j + 1) ^ sw) << 4), make_uint4(codes[4], codes[5], codes[6], codes[7]));
                    sft[(j >> 2) * 512 + row * 16 + (j & 3)] = static_cast<uint8_t>(sc);
                } else if constexpr (KIND == 1) {  // NVFP4: 16 bytes of codes, scale blocks 2j and 2j + 1
                    st_shared_v4(t_row + ((j ^ sw) << 4), make_uint4(codes[0], codes[1], codes[2], codes[3]));
                    *reinterpret_cast<uint16_t*>(sft + ((2 * j) >> 2) * 512 + row * 16 + ((2 * j) & 3)) =
                        static_cast<uint16_t>(sc);
                } else {  // MXFP4: 16 bytes of codes, one scale block
                    st_shared_v4(t_row + ((j ^ sw) << 4), make_uint4(codes[0], codes[1], codes[2], codes[3]));
                    sft[(j >> 2) * 512 + row * 16 + (j & 3)] = static_cast<uint8_t>(sc);
                }
            }
            fence_proxy_async_smem();  // the token tile is read next by the tensor core
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&tready[ts]);
                mbar_arrive(&xempty[xs]);
            }
            if (++xs == XS) {
                xs = 0;
                xph ^= 1u;
            }
            if (++ts == TS) {
                ts = 0;
                tph ^= 1u;
            }
        }
    }

    // reduction and epilogue: warp w of 3-10 holds the 16 tokens [16 h, +16) (h = (w - 3) / 4) of the
    // 32 weight rows in its TMEM sub-partition, for each weight group.  With a K split (WG = 1) the
    // non-leaders send their partials to the leader's buffer ([split - 1][token quad][128 rows][4]
    // fp32: a warp's 16-byte stores cover 512 contiguous bytes) as soon as their MMAs are done, and
    // the leader adds them in split order.
    const bool epi = warp >= 3;
    const int sub = warp & 3;
    const int h = (warp - 3) >> 2;
    const int wrow = sub * 32 + lane;  // weight row within a 128-row group
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
    float acc[WG][16];
    cluster_wait();  // every CTA of the cluster has initialised its barriers
    if (epi) {
        const bool ok = mbar_wait(accf, 0, p.status, 57);
        tc_fence_after();
#pragma unroll
        for (int g = 0; g < WG; ++g) {
            uint32_t r[16];
            tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + static_cast<uint32_t>(g * C::TOK + 16 * h),
                               r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[g][i] = ok ? __uint_as_float(r[i]) : 0.0f;
        }
        tc_fence_before();
    }
    if constexpr (WG == 1) {
        if (epi && split != 0) {
            const uint32_t dst = mapa_shared(smem_u32(red + (((split - 1) * (C::TOK / 4) + 4 * h) * 128 + wrow) * 4), 0);
            const uint32_t bar = mapa_shared(smem_u32(rfull), 0);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                st_async_v4(dst + q * 128 * 16, acc[0][4 * q], acc[0][4 * q + 1], acc[0][4 * q + 2], acc[0][4 * q + 3],
                            bar);
        }
    }
    if (epi && split == 0) {
        const bool got = mbar_wait(rfull, 0, p.status, 58);
        if constexpr (WG == 1) {
            for (uint32_t sp = 1; got && sp < splits; ++sp) {
                const float4* src = reinterpret_cast<const float4*>(red) + ((sp - 1) * (C::TOK / 4) + 4 * h) * 128 + wrow;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 v = src[q * 128];
                    acc[0][4 * q] = __fadd_rn(acc[0][4 * q], v.x);
                    acc[0][4 * q + 1] = __fadd_rn(acc[0][4 * q + 1], v.y);
                    acc[0][4 * q + 2] = __fadd_rn(acc[0][4 * q + 2], v.z);
                    acc[0][4 * q + 3] = __fadd_rn(acc[0][4 * q + 3], v.w);
                }
            }
        }
        const float alpha = (KIND == 1) ? __fmul_rn(*p.g_a, *p.g_b) : 1.0f;
        if (!OUT_F32 && p.tma_store) {
            // each group's [32 tokens][128 columns] bf16 tile through shared memory (the token ring is
            // idle now: every stage has been quantized) and one TMA store, clipped at the M and N
            // edges; direct stores would write one 2-byte element per token row and lane
#pragma unroll
            for (int g = 0; g < WG; ++g) {
                uint16_t* stg = reinterpret_cast<uint16_t*>(smem + C::OFF_X) + g * C::TOK * 128;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float v = KIND == 1 ? __fmul_rn(acc[g][i], alpha) : acc[g][i];
                    stg[(16 * h + i) * 128 + wrow] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
                }
            }
            fence_proxy_async_smem();
            named_barrier_sync(2, 32 * C::QWARPS);
            if (warp == 3 && lane == 0) {
                for (int g = 0; g < WG; ++g) {
                    if ((nt * WG + g) * 128 >= p.N) break;
                    tma_store_2d(&tma_out, reinterpret_cast<uint16_t*>(smem + C::OFF_X) + g * C::TOK * 128,
                                 (nt * WG + g) * 128, 0);
                    bulk_commit_group();
                }
                bulk_wait_group0();
            }
        } else {
#pragma unroll
            for (int g = 0; g < WG; ++g) {
                const int n = (nt * WG + g) * 128 + wrow;
                if (n >= p.N) continue;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int m = 16 * h + i;
                    if (m < p.M) {
                        const float v = KIND == 1 ? __fmul_rn(acc[g][i], alpha) : acc[g][i];
                        if constexpr (OUT_F32) {
                            static_cast<float*>(p.out)[static_cast<int64_t>(m) * p.N + n] = v;
                        } else {
                            static_cast<__nv_bfloat16*>(p.out)[static_cast<int64_t>(m) * p.N + n] = __float2bfloat16_rn(v);
                        }
                    }
                }
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ small-N linear kernel
//
// Linear layers with few output columns (N <= 128, e.g. a fused N = 96 projection) and many
// tokens.  With one column tile the GEMM reads every activation row exactly once, so it quantizes
// the bf16 rows itself instead of reading codes that a separate quantizer pass wrote: A crosses
// HBM once, as bf16, and no codes round-trip through it.  One CTA per 128-row M tile and K split;
// the S CTAs of a cluster split the K stages and reduce their partial accumulators through
// distributed shared memory in the leader, as the split-K kernel does.  The bf16 rows stream
// through a ring of 16 KB slots (64 elements x 128 rows, 128B swizzle) deeper than the stages the
// tensor cores consume, so that about 128 KB per SM stay in flight from HBM.
//   warp 0       TMA producer of the bf16 slots
//   warp 1       TMEM owner; copies the stage's scale tiles into TMEM (tcgen05.cp), issues the MMAs
//   warp 2       TMA producer of the weight stages (codes 128 rows x 128 bytes, scale tiles)
//   warps 3-18   quantize each stage's rows into the A tile (codes in the 128B-swizzled operand
//                layout, scales in the 512-byte tile layout) with the streaming quantizer's
//                arithmetic (16 warps: the quantization is latency-bound per warp); after the last
//                stage they are the epilogue, which stores through shared memory and TMA
template <int KIND>
struct RowqCfg {
    static constexpr int BS = Fmt<KIND>::BS, EPB = Fmt<KIND>::EPB, MMA_K = Fmt<KIND>::MMA_K;
    static constexpr int BK = 128 * EPB;          // K elements per stage: 128 code bytes per row
    static constexpr int KSTEPS = BK / MMA_K;     // 4 MMAs per stage
    static constexpr int KB_PER_MMA = MMA_K / BS;
    static constexpr int SF_ATOMS = BK / BS / 4;  // 512-byte scale tiles per 128 rows per stage
    static constexpr int BN = 128;
    static constexpr int XSLOTS = 8;              // bf16 slots of 64 elements x 128 rows
    static constexpr int XPS = BK / 64;           // slots per stage (4 FP4, 2 MXFP8), one barrier per stage
    static constexpr int XSTAGES = XSLOTS / XPS;
    static constexpr int ASTAGES = 2, BSTAGES = 2;
    static constexpr int X_BYTES = 128 * 128;
    static constexpr int A_BYTES = 128 * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int SF_BYTES = SF_ATOMS * 512;
    static constexpr int QWARPS = 16;
    static constexpr int THREADS = (3 + QWARPS) * 32;
    static constexpr int OFF_X = 0;
    static constexpr int OFF_A = OFF_X + XSLOTS * X_BYTES;
    static constexpr int OFF_B = OFF_A + ASTAGES * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + BSTAGES * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + ASTAGES * SF_BYTES;
    static constexpr int OFF_TAB = OFF_SFB + BSTAGES * SF_BYTES;  // NVFP4 d and 1/d per scale code
    static constexpr int OFF_BAR = OFF_TAB + 1024;
    static constexpr int N_BARS = 2 * (XSTAGES + ASTAGES + BSTAGES) + 3;  // + accf, rready, rfull
    static constexpr int OFF_SLOT = OFF_BAR + N_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_SLOT + 16 + 1024;
    static constexpr int SLOT_COLS = 2 * SF_ATOMS * 4;  // per B stage: A then B scale tiles
    static constexpr int SF_TMEM_BASE = BN;
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr int STG_BYTES = 32 * 64;           // per epilogue warp: 32 rows x 32 bf16 columns
    static_assert(KSTEPS == 4, "4 MMAs per stage");
    static_assert(XSLOTS % XPS == 0, "whole stages in the bf16 ring");
    static_assert(SF_TMEM_BASE + BSTAGES * SLOT_COLS <= static_cast<int>(TMEM_COLS), "TMEM budget");
    static_assert((kMaxSplits - 1) * 128 * BN * 4 <= OFF_TAB, "reduction buffer inside the rings");
    static constexpr int EARLY_SPLITS = XSLOTS * X_BYTES / (128 * BN * 4) + 1;  // partials inside the bf16 ring
    static_assert(EARLY_SPLITS >= 2, "at least one partial fits in the bf16 ring");
    static_assert(QWARPS * STG_BYTES <= OFF_TAB, "output staging inside the rings");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <int KIND, bool OUT_F32, int QRULE>
__global__ void __launch_bounds__(RowqCfg<KIND>::THREADS, 1)
    gemm_rowq_kernel(const __grid_constant__ CUtensorMap tma_x, const __grid_constant__ CUtensorMap tma_b,
                     const __grid_constant__ CUtensorMap tma_out, const GemmArgs p) {
    using C = RowqCfg<KIND>;
    constexpr int BN = C::BN, AS = C::ASTAGES, BSt = C::BSTAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* xfull = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* xempty = xfull + C::XSTAGES;
    uint64_t* aready = xempty + C::XSTAGES;
    uint64_t* aempty = aready + AS;
    uint64_t* bfull = aempty + AS;
    uint64_t* bempty = bfull + BSt;
    uint64_t* accf = bempty + BSt;
    uint64_t* rready = accf + 1;  // non-leaders: the leader's rings are free for the partials
    uint64_t* rfull = accf + 2;   // leader: every partial has landed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_SLOT);
    float* tab_d = reinterpret_cast<float*>(smem + C::OFF_TAB);
    float* tab_r = tab_d + 128;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t split = cluster_ctarank();
    const uint32_t splits = p.k_split;
    const int mt = static_cast<int>(blockIdx.x / splits);
    const int mrows = min(128, p.M - mt * 128);  // valid rows of this M tile
    const int per = (p.k_stages + static_cast<int>(splits) - 1) / static_cast<int>(splits);
    const int k0 = static_cast<int>(split) * per;
    const int k1 = min(p.k_stages, k0 + per);
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tma_x);
        prefetch_tmap(&tma_b);
        for (int s = 0; s < C::XSTAGES; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&xempty[s], C::QWARPS);
        }
        for (int s = 0; s < AS; ++s) {
            mbar_init(&aready[s], C::QWARPS);
            mbar_init(&aempty[s], 1);
        }
        for (int s = 0; s < BSt; ++s) {
            mbar_init(&bfull[s], 1);
            mbar_init(&bempty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(rready, 1);
        mbar_init(rfull, 1);
        // the partials of the other CTAs: valid rows, and only the 32-column groups below N
        const uint32_t groups = static_cast<uint32_t>(min(BN, (p.N + 31) & ~31) / 32);
        if (split == 0) mbar_arrive_expect_tx(rfull, (splits - 1) * static_cast<uint32_t>(mrows) * groups * 32 * 4);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_arrive_relaxed();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();
    pdl_launch_dependents();  // the next kernel on the stream may start its prologue

    if (warp == 0) {
        // bf16 producer: the XPS 64-element boxes of a stage land in slots xs * XPS + b and complete
        // on one barrier (a barrier per box made this one thread's loads complete about one at a
        // time, 0.5 us per 16 KB box from HBM)
        const uint64_t pol = policy_evict_first();
        int xs = 0;
        uint32_t phase = 0;
        for (int ks = k0; ks < k1; ++ks) {
            if (!mbar_wait_warp(&xempty[xs], phase ^ 1u, p.status, 41)) break;
            if (elect_one()) {
                mbar_arrive_expect_tx(&xfull[xs], C::XPS * C::X_BYTES);
#pragma unroll
                for (int b = 0; b < C::XPS; ++b)
                    tma_load_2d(&tma_x, &xfull[xs], smem + C::OFF_X + (xs * C::XPS + b) * C::X_BYTES,
                                (ks * C::BK + b * 64) * 2, mt * 128, pol);
            }
            __syncwarp();
            if (++xs == C::XSTAGES) {
                xs = 0;
                phase ^= 1u;
            }
        }
    } else if (warp == 2) {
        // weight producer
        const uint64_t pol = policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        for (int ks = k0; ks < k1; ++ks) {
            if (!mbar_wait_warp(&bempty[stage], phase ^ 1u, p.status, 48)) break;
            if (elect_one()) {
                const int atoms = min(C::SF_ATOMS, p.sf_col_tiles - ks * C::SF_ATOMS);
                mbar_arrive_expect_tx(&bfull[stage], C::B_BYTES + atoms * 512);
                tma_load_2d(&tma_b, &bfull[stage], smem + C::OFF_B + stage * C::B_BYTES, ks * 128, 0, pol);
                bulk_load(smem + C::OFF_SFB + stage * C::SF_BYTES,
                          p.b_sf + static_cast<int64_t>(ks) * C::SF_ATOMS * 512, atoms * 512, &bfull[stage]);
            }
            __syncwarp();
            if (++stage == BSt) {
                stage = 0;
                phase ^= 1u;
            }
        }
    } else if (warp == 1) {
        // scale copies and MMAs: the whole warp runs the loop; one elected lane issues
        int as = 0, bs = 0;
        uint32_t aph = 0, bph = 0;
        bool ok = true;
        for (int ks = k0; ks < k1; ++ks) {
            if (!mbar_wait_warp(&bfull[bs], bph, p.status, 42) || !mbar_wait_warp(&aready[as], aph, p.status, 43)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // TMEM scale slot of this B stage (free: its previous MMAs completed before the
            // producer could refill the stage)
            const uint32_t sf_col = tmem_base + C::SF_TMEM_BASE + bs * C::SLOT_COLS;
            const uint32_t sfa_s = smem_u32(smem + C::OFF_SFA + as * C::SF_BYTES);
            const uint32_t sfb_s = smem_u32(smem + C::OFF_SFB + bs * C::SF_BYTES);
            const uint32_t a_s = smem_u32(smem + C::OFF_A + as * C::A_BYTES);
            const uint32_t b_s = smem_u32(smem + C::OFF_B + bs * C::B_BYTES);
            if (elect_one()) {
#pragma unroll
                for (int a = 0; a < C::SF_ATOMS; ++a) {
                    tc_cp_scales(sf_col + a * 4, smem_desc(sfa_s + a * 512, 0, 128, kLayoutNone));
                    tc_cp_scales(sf_col + C::SF_ATOMS * 4 + a * 4, smem_desc(sfb_s + a * 512, 0, 128, kLayoutNone));
                }
#pragma unroll
                for (int j = 0; j < C::KSTEPS; ++j) {
                    if (ks * C::BK + j * C::MMA_K < p.K) {
                        const int kb = j * C::KB_PER_MMA;
                        const int atom = kb >> 2;
                        mma_block_scaled<KIND>(tmem_base, smem_desc(a_s + j * 32, 16, 1024, kLayoutSwizzle128B),
                                               smem_desc(b_s + j * 32, 16, 1024, kLayoutSwizzle128B),
                                               mma_idesc<KIND>(kBM, BN, static_cast<uint32_t>(kb & 3)),
                                               sf_col + atom * 4, sf_col + C::SF_ATOMS * 4 + atom * 4,
                                               (ks > k0 || j > 0) ? 1u : 0u);
                    }
                }
                tc_commit(&aempty[as]);
                tc_commit(&bempty[bs]);
            }
            __syncwarp();
            if (++as == AS) {
                as = 0;
                aph ^= 1u;
            }
            if (++bs == BSt) {
                bs = 0;
                bph ^= 1u;
            }
        }
        if (ok && elect_one()) tc_commit(accf);
        __syncwarp();
    } else {
        // quantizers: thread qt takes units (row, j) of 32 elements, a warp 32 consecutive rows of
        // one unit column, so its 16-byte reads of the swizzled bf16 rows fall in distinct banks
        const int qt = (warp - 3) * 32 + lane;
        constexpr int UPR = C::BK / 32;                    // units per row and stage
        constexpr int UPT = 128 * UPR / (32 * C::QWARPS);  // units per thread and stage
        static_assert(128 * UPR % (32 * C::QWARPS) == 0, "whole units per thread");
        float g_a = 1.0f;
        if constexpr (KIND == 1) {
            g_a = *p.g_a;
            if (qt < 128) {
                const float d = __fmul_rn(e4m3_decode_pos(static_cast<uint32_t>(qt)), g_a);
                tab_d[qt] = d;
                tab_r[qt] = __frcp_rn(d);  // fl(1/d), +inf for d = 0
            }
            named_barrier_sync(1, 32 * C::QWARPS);
        }
        int xs = 0, as = 0;
        uint32_t xph = 0, aph = 0;
        bool ok = true;
        for (int ks = k0; ks < k1 && ok; ++ks) {
            ok = mbar_wait_warp(&xfull[xs], xph, p.status, 44);
            if (!ok || !mbar_wait_warp(&aempty[as], aph ^ 1u, p.status, 49)) break;
            const uint32_t a_s = smem_u32(smem + C::OFF_A + as * C::A_BYTES);
            uint8_t* sfa = smem + C::OFF_SFA + as * C::SF_BYTES;
#pragma unroll
            for (int u = 0; u < UPT; ++u) {
                const int v = qt + u * 32 * C::QWARPS;
                const int row = v & 127, j = v >> 7;
                if (static_cast<int64_t>(ks) * C::BK + j * 32 >= p.K) continue;
                uint32_t w[16];
                const uint32_t rb = smem_u32(smem + C::OFF_X + (xs * C::XPS + (j >> 1)) * C::X_BYTES) + row * 128;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 t = ld_shared_v4(rb + ((((j & 1) * 4 + i) ^ (row & 7)) << 4));
                    w[4 * i] = t.x;
                    w[4 * i + 1] = t.y;
                    w[4 * i + 2] = t.z;
                    w[4 * i + 3] = t.w;
                }
                uint32_t codes[8], seen = 0;
                const uint32_t sc = quantize32<KIND, (QRULE < 0 ? 0 : QRULE), false>(w, g_a, tab_d, tab_r, codes, seen);
                const uint32_t sw = static_cast<uint32_t>(row & 7);
                const uint32_t sf_row = (row & 31) * 16 + ((row >> 5) & 3) * 4;
                const uint32_t a_row = a_s + row * 128;
                if constexpr (KIND == 2) {  // MXFP8: 32 bytes of codes, one scale block
                    st_shared_v4(a_row + (((2 * j) ^ sw) << 4), make_uint4(codes[0], codes[1], codes[2], codes[3]));
                    st_shared_v4(a_row + (((2 * j + 1) ^ sw) << 4), make_uint4(codes[4], codes[5], codes[6], codes[7]));
                    sfa[(j >> 2) * 512 + sf_row + (j & 3)] = static_cast<uint8_t>(sc);
                } else if constexpr (KIND == 1) {  // NVFP4: 16 bytes of codes, scale blocks 2j and 2j + 1
                    st_shared_v4(a_row + ((j ^ sw) << 4), make_uint4(codes[0], codes[1], codes[2], codes[3]));
                    *reinterpret_cast<uint16_t*>(sfa + ((2 * j) >> 2) * 512 + sf_row + ((2 * j) & 3)) =
                        static_cast<uint16_t>(sc);
                } else {  // MXFP4: 16 bytes of codes, one scale block
                    st_shared_v4(a_row + ((j ^ sw) << 4), make_uint4(codes[0], codes[1], codes[2], codes[3]));
                    sfa[(j >> 2) * 512 + sf_row + (j & 3)] = static_cast<uint8_t>(sc);
                }
            }
            fence_proxy_async_smem();  // the A tile and scale tiles are read next by the tensor core
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&aready[as]);
                mbar_arrive(&xempty[xs]);
            }
            if (++xs == C::XSTAGES) {
                xs = 0;
                xph ^= 1u;
            }
            if (++as == AS) {
                as = 0;
                aph ^= 1u;
            }
        }
        // with up to EARLY_SPLITS CTAs the partials land in the leader's bf16 ring only, which is
        // idle once every quantizer warp is done with the last stage: the leader lets the other
        // CTAs send them now, while its last MMAs still run, instead of after them
        if (split == 0 && splits > 1 && splits <= static_cast<uint32_t>(C::EARLY_SPLITS)) {
            cluster_wait();  // the other CTAs' barriers are initialised (these warps wait here, not below)
            named_barrier_sync(3, 32 * C::QWARPS);
            if (warp == 3 && lane == 0)
                for (uint32_t sp = 1; sp < splits; ++sp) mbar_arrive_cluster(mapa_shared(smem_u32(rready), sp));
        }
    }

    // reduction and epilogue: warps 3-18 hold 32 accumulator columns of one TMEM sub-partition
    // each; the leader frees its rings for the partials (its bf16 ring once its quantizers are done
    // with it, for up to EARLY_SPLITS CTAs; else its rings once its MMAs are done), the others send
    // their valid rows with st.async (column-quad-major layout, as in the split-K kernel) and
    // leave; the leader adds them in split order and stores through a staging tile per warp and a
    // TMA store (rows per lane, so direct stores would touch one sector per element)
    constexpr int COLS = BN / (C::QWARPS / 4);
    const bool epi = warp >= 3;
    const int sub = warp & 3;
    const int col0 = ((warp - 3) >> 2) * COLS;
    const int row = sub * 32 + lane;
    float* red = reinterpret_cast<float*>(smem);
    float acc[COLS];
    const bool early = split == 0 && splits > 1 && splits <= static_cast<uint32_t>(C::EARLY_SPLITS);
    if (!(epi && early)) cluster_wait();  // every CTA of the cluster has initialised its barriers
    if (epi) {
        const bool ok = mbar_wait(accf, 0, p.status, 45);
        if (split == 0 && splits > static_cast<uint32_t>(C::EARLY_SPLITS) && warp == 3 && lane == 0)
            for (uint32_t sp = 1; sp < splits; ++sp) mbar_arrive_cluster(mapa_shared(smem_u32(rready), sp));
        tc_fence_after();
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) + static_cast<uint32_t>(col0);
#pragma unroll
        for (int c = 0; c < COLS / 32; ++c) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_row + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[c * 32 + i] = ok ? __uint_as_float(r[i]) : 0.0f;
        }
        tc_fence_before();
    }
    static_assert(COLS == 32, "one 32-column group per epilogue warp");
    if (epi && split != 0 && row < mrows && col0 < p.N && mbar_wait_cluster(rready, 0, p.status, 46)) {
        const uint32_t dst = mapa_shared(smem_u32(red + (((split - 1) * (BN / 4) + col0 / 4) * 128 + row) * 4), 0);
        const uint32_t bar = mapa_shared(smem_u32(rfull), 0);
#pragma unroll
        for (int v = 0; v < COLS / 4; ++v)
            st_async_v4(dst + v * 128 * 16, acc[4 * v], acc[4 * v + 1], acc[4 * v + 2], acc[4 * v + 3], bar);
    }
    if (epi && split == 0) {
        const bool got = row < mrows ? mbar_wait(rfull, 0, p.status, 47) : true;
        for (uint32_t sp = 1; got && row < mrows && col0 < p.N && sp < splits; ++sp) {
            const float4* src = reinterpret_cast<const float4*>(red) + ((sp - 1) * (BN / 4) + col0 / 4) * 128 + row;
#pragma unroll
            for (int v = 0; v < COLS / 4; ++v) {
                const float4 q = src[v * 128];
                acc[4 * v] = __fadd_rn(acc[4 * v], q.x);
                acc[4 * v + 1] = __fadd_rn(acc[4 * v + 1], q.y);
                acc[4 * v + 2] = __fadd_rn(acc[4 * v + 2], q.z);
                acc[4 * v + 3] = __fadd_rn(acc[4 * v + 3], q.w);
            }
        }
        const float alpha = (KIND == 1) ? __fmul_rn(*p.g_a, *p.g_b) : 1.0f;
        const int64_t m = static_cast<int64_t>(mt) * 128 + row;
        if constexpr (!OUT_F32) {
            uint32_t packed[COLS / 2];
#pragma unroll
            for (int i = 0; i < COLS / 2; ++i) {
                const float lo = KIND == 1 ? __fmul_rn(acc[2 * i], alpha) : acc[2 * i];
                const float hi = KIND == 1 ? __fmul_rn(acc[2 * i + 1], alpha) : acc[2 * i + 1];
                const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
                packed[i] = *reinterpret_cast<const uint32_t*>(&b);
            }
            if (p.tma_store) {
                // every epilogue warp is done reading the partials before the staging tiles reuse them;
                // lanes past the last valid row skipped the waits above, and bar.sync wants whole warps
                __syncwarp();
                named_barrier_sync(2, 32 * C::QWARPS);
                // 32 rows x 32 columns per warp, 64B swizzle (16-byte piece q of row r at q ^ ((r >> 1) & 3))
                uint8_t* stg = smem + (warp - 3) * C::STG_BYTES;
                const uint32_t st_row = smem_u32(stg) + lane * 64;
                const uint32_t sw = static_cast<uint32_t>((lane >> 1) & 3);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    st_shared_v4(st_row + ((q ^ sw) << 4),
                                 make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]));
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && sub * 32 < mrows && col0 < p.N) {
                    tma_store_2d(&tma_out, stg, col0, mt * 128 + sub * 32);  // clipped at the M and N edges
                    bulk_commit_group();
                    bulk_wait_group0();
                }
            } else if (row < mrows) {
                uint16_t* o16 = reinterpret_cast<uint16_t*>(p.out) + m * p.N;
#pragma unroll
                for (int i = 0; i < COLS / 2; ++i) {
                    const int n = col0 + 2 * i;
                    if (n < p.N) o16[n] = static_cast<uint16_t>(packed[i] & 0xFFFFu);
                    if (n + 1 < p.N) o16[n + 1] = static_cast<uint16_t>(packed[i] >> 16);
                }
            }
        } else if (row < mrows) {
            float* orow = static_cast<float*>(p.out) + m * p.N;
#pragma unroll
            for (int i = 0; i < COLS; ++i)
                if (col0 + i < p.N) orow[col0 + i] = __fmul_rn(acc[i], alpha);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ CTA-pair kernel
//
// Two CTAs of a cluster on two SMs compute one 256 x BN tile with cta_group::2 MMAs: CTA r loads
// A rows [128 r, +128) and B rows [BN/2 r, +BN/2) of the tile, so each SM streams 128 rows of A
// and BN/2 rows of B per 128-byte K slice.  Every load of both CTAs (operands, the CTA's own A
// scale tiles and the scale tiles of all the tile's B rows) is a TMA load that completes on the
// leader's barrier; the leader's MMA warp then copies both CTAs' scale tiles into their TMEM
// (tcgen05.cp.cta_group::2, each CTA from its own shared memory) and issues the stage's MMAs
// behind them in the tensor pipe.  The only cross-CTA signals per stage are the TMA completions
// and the MMA commit multicast to both CTAs.  (A separate scale-copy warp with a barrier of its
// own put one more hop into every stage's round trip and measured 1-2 % slower.)
//
// A stage slot's round trip (reissued -> its data landed 1.5 us -> MMAs issued 0.2 us -> MMAs done
// and the slot reissued 0.6 us) is about 2.2 us, with all SMs together pulling about 11.5 TB/s of
// operands out of L2.  Without the operand loads the kernel runs at 6.9 PFLOP/s (MXFP4): each
// block-scaled pair MMA costs about 0.085 us whether N is 256 or 128, so a 256 x 384 tile (an N =
// 256 and an N = 128 MMA per K step, 17 % fewer operand bytes per FLOP) measured slower.
//
// BN = 256 keeps one accumulator (256 TMEM columns + the scale slots fill the 512), so the
// tensor pipe idles while the epilogue drains it at every tile boundary.  BN = 192 fits two
// accumulators (2 x 192 + 5 x 24 scale columns): the epilogue drains one while the MMAs fill the
// other.  A 192-row tile starts 0 or 64 rows into a 128-row scale tile; the MMA then addresses
// the B scales 0 or 2 TMEM columns into the two copied scale tiles (32 rows per column).
//   warp 0       TMA producer (both CTAs)
//   warp 1       TMEM owner (both CTAs); scale copies and MMA issuer (leader)
//   warps 2-     epilogue (both CTAs): EPI_WARPS / 4 warps per TMEM sub-partition, COLS columns each
// The single-thread roles run as converged warps that issue through one elected lane.

template <int KIND, int STAGES, int BN>
struct PairCfg {
    static_assert(BN == 256 || BN == 192, "pair tile width");
    static constexpr int BS = Fmt<KIND>::BS, EPB = Fmt<KIND>::EPB, MMA_K = Fmt<KIND>::MMA_K;
    static constexpr int BK = 128 * EPB;
    static constexpr int KSTEPS = BK / MMA_K;
    static constexpr int KB_PER_MMA = MMA_K / BS;
    static constexpr int SF_ATOMS = BK / BS / 4;
    static constexpr int ACC = (BN == 256) ? 1 : 2;    // accumulator buffers
    static constexpr int B_ROWS = BN / 2;              // B rows per CTA
    static constexpr int COLS = (BN == 256) ? 128 : 64;  // accumulator columns per epilogue warp
    static constexpr int EPI_WARPS = 4 * (BN / COLS);
    static constexpr int THREADS = (2 + EPI_WARPS) * 32;
    static constexpr int A_BYTES = 128 * 128;
    static constexpr int B_BYTES = B_ROWS * 128;
    static constexpr int SFA_BYTES = SF_ATOMS * 512;
    static constexpr int SFB_BYTES = 2 * SF_ATOMS * 512;  // the tile's B rows lie in two 128-row scale tiles
    static constexpr int CTA_STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int SF_COLS_A = SF_ATOMS * 4;
    static constexpr int SF_COLS_B = SF_ATOMS * 8;
    static constexpr int SF_COLS_STAGE = SF_COLS_A + SF_COLS_B;
    static constexpr int SF_TMEM_BASE = ACC * BN;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(SF_TMEM_BASE + STAGES * SF_COLS_STAGE <= 512, "TMEM budget");
    static_assert(KSTEPS == 4, "4 MMAs per 128-byte stage");
    static_assert(B_BYTES % 1024 == 0, "128B-swizzled operand buffers stay 1024-byte aligned");
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
    // epilogue staging for TMA stores: one 32-row x 64-column bf16 tile (4 KB, 128B-swizzled) per warp
    static constexpr int STG_BYTES = 4096;
    static constexpr int OFF_STG = ((OFF_SFB + STAGES * SFB_BYTES) + 1023) / 1024 * 1024;
    static constexpr int OFF_BAR = OFF_STG + EPI_WARPS * STG_BYTES;
    static constexpr int N_BARS = 2 * STAGES + 2 * ACC;
    static constexpr int OFF_SLOT = OFF_BAR + N_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_SLOT + 16 + 1024;
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <int KIND, int STAGES, int BN, bool OUT_F32>
__global__ void __launch_bounds__(PairCfg<KIND, STAGES, BN>::THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                     const __grid_constant__ CUtensorMap tma_sfa, const __grid_constant__ CUtensorMap tma_sfb,
                     const __grid_constant__ CUtensorMap tma_out, const GemmArgs p) {
    using C = PairCfg<KIND, STAGES, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);  // leader: all loads of both CTAs landed
    uint64_t* empty = full + STAGES;                                   // both: the stage's MMAs are done
    uint64_t* accf = empty + STAGES;                                   // both: accumulator buffer ready
    uint64_t* acce = accf + C::ACC;                                    // leader: accumulator buffer drained by both
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_SLOT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = static_cast<int>(blockIdx.x >> 1), num_pairs = static_cast<int>(gridDim.x >> 1);
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tma_a);
        prefetch_tmap(&tma_b);
        prefetch_tmap(&tma_sfa);
        prefetch_tmap(&tma_sfb);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < C::ACC; ++a) {
            mbar_init(&accf[a], 1);
            mbar_init(&acce[a], 2 * C::EPI_WARPS);
        }
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    pdl_wait();
    pdl_launch_dependents();  // the next kernel on the stream may start its prologue

    const int m_tiles = (p.M + 255) / 256;
    const int num_tiles = m_tiles * p.n_tiles;
    if (warp == 0) {
        // TMA producer: the whole warp runs the loop; one elected lane issues
        const uint64_t pol_a = policy_evict_last();
        const uint64_t pol_b = policy_evict_normal();
        const uint32_t full_leader = mapa_shared(smem_u32(full), 0);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
            int mt, nt;
            pair_tile_coords(tile, m_tiles, p.n_tiles, p.group_m, mt, nt);
            const int a_row = (2 * mt + static_cast<int>(rank)) * 128;            // this CTA's A rows
            const int b_row = nt * BN + static_cast<int>(rank) * C::B_ROWS;       // this CTA's B rows
            const int sf_b_tile = (nt * BN) >> 7;  // first 128-row scale tile of the tile's B rows
            for (int ks = 0; ks < p.k_stages; ++ks) {
                if (!mbar_wait_warp(&empty[stage], phase ^ 1u, p.status, 11)) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::CTA_STAGE_BYTES);
                    const uint32_t fb = full_leader + stage * 8;
                    tma_load_2d_pair(&tma_a, fb, smem + C::OFF_A + stage * C::A_BYTES, ks * 128, a_row, pol_a);
                    tma_load_2d_pair(&tma_b, fb, smem + C::OFF_B + stage * C::B_BYTES, ks * 128, b_row, pol_b);
                    // scale tiles: rows of 256 bytes (half a 512-byte tile); a box covers SF_ATOMS tiles
                    const int kcol = ks * C::SF_ATOMS;
                    tma_load_2d_pair(&tma_sfa, fb, smem + C::OFF_SFA + stage * C::SFA_BYTES, 0,
                                     ((a_row >> 7) * p.sf_col_tiles + kcol) * 2, pol_a);
#pragma unroll
                    for (int g = 0; g < 2; ++g)
                        tma_load_2d_pair(&tma_sfb, fb, smem + C::OFF_SFB + stage * C::SFB_BYTES + g * C::SF_ATOMS * 512,
                                         0, ((sf_b_tile + g) * p.sf_col_tiles + kcol) * 2, pol_b);
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        if (rank == 0) {
            // MMA issuer (leader): the whole warp runs the loop; one elected lane issues
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
                int mt, nt;
                pair_tile_coords(tile, m_tiles, p.n_tiles, p.group_m, mt, nt);
                const uint32_t sfb_shift = static_cast<uint32_t>(((nt * BN) & 127) >> 5);  // 0, or 2 for BN = 192
                if (!mbar_wait_warp(&acce[acc], acc_phase ^ 1u, p.status, 12)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int ks = 0; ks < p.k_stages; ++ks) {
                    if (!mbar_wait_warp(&full[stage], phase, p.status, 13)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sf_col = tmem_base + C::SF_TMEM_BASE + stage * C::SF_COLS_STAGE;
                    const uint32_t a_s = smem_u32(smem + C::OFF_A + stage * C::A_BYTES);
                    const uint32_t b_s = smem_u32(smem + C::OFF_B + stage * C::B_BYTES);
                    const uint32_t sfa_s = smem_u32(smem + C::OFF_SFA + stage * C::SFA_BYTES);
                    const uint32_t sfb_s = smem_u32(smem + C::OFF_SFB + stage * C::SFB_BYTES);
                    if (elect_one()) {
                        // this stage's scale tiles into both CTAs' TMEM, ahead of its MMAs in the
                        // tensor pipe (the slot's previous MMAs completed before its loads were issued)
#pragma unroll
                        for (int a = 0; a < C::SF_ATOMS; ++a) {
                            tc_cp_scales_pair(sf_col + a * 4, smem_desc(sfa_s + a * 512, 0, 128, kLayoutNone));
#pragma unroll
                            for (int g = 0; g < 2; ++g)
                                tc_cp_scales_pair(sf_col + C::SF_COLS_A + a * 8 + g * 4,
                                                  smem_desc(sfb_s + (g * C::SF_ATOMS + a) * 512, 0, 128, kLayoutNone));
                        }
#pragma unroll
                        for (int j = 0; j < C::KSTEPS; ++j) {
                            if (ks * C::BK + j * C::MMA_K < p.K) {
                                const int kb = j * C::KB_PER_MMA;
                                const int atom = kb >> 2;
                                const uint32_t idesc = mma_idesc<KIND>(256, BN, static_cast<uint32_t>(kb & 3));
                                mma_block_scaled_pair<KIND>(d_tmem, smem_desc(a_s + j * 32, 16, 1024, kLayoutSwizzle128B),
                                                            smem_desc(b_s + j * 32, 16, 1024, kLayoutSwizzle128B), idesc,
                                                            sf_col + atom * 4, sf_col + C::SF_COLS_A + atom * 8 + sfb_shift,
                                                            (ks | j) != 0 ? 1u : 0u);
                            }
                        }
                        tc_commit_pair(&empty[stage], 0x3);
                    }
                    __syncwarp();
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (elect_one()) tc_commit_pair(&accf[acc], 0x3);
                __syncwarp();
                if (++acc == C::ACC) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
        }
    } else {
        constexpr int COLS = C::COLS;  // accumulator columns owned by this warp
        const int sub = warp & 3;
        const int col0 = ((warp - 2) >> 2) * COLS;
        const int row = sub * 32 + lane;
        const float alpha = (KIND == 1) ? __fmul_rn(*p.g_a, *p.g_b) : 1.0f;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = pair; tile < num_tiles; tile += num_pairs) {
            int mt, nt;
            pair_tile_coords(tile, m_tiles, p.n_tiles, p.group_m, mt, nt);
            const uint32_t acce_leader = mapa_shared(smem_u32(&acce[acc]), 0);
            if (!mbar_wait(&accf[acc], acc_phase, p.status, 14)) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(sub * 32) << 16) +
                                   static_cast<uint32_t>(acc * BN + col0);
            const int m = mt * 256 + static_cast<int>(rank) * 128 + row;
            const int n0 = nt * BN + col0;
            if constexpr (!OUT_F32) {
                __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(m) * p.N;
                const bool vec = (n0 + COLS <= p.N) && (p.N & 7) == 0;
                // drain this warp's columns into registers (two TMEM loads per wait), release the
                // accumulator, then store: the stores overlap the MMAs of the next tile
                uint32_t packed[COLS / 2];
#pragma unroll
                for (int c = 0; c < COLS / 32; c += 2) {
                    uint32_t r0[32], r1[32];
                    tmem_ld_32x32b_x32(t_row + c * 32, r0);
                    tmem_ld_32x32b_x32(t_row + c * 32 + 32, r1);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float lo = __uint_as_float(r0[2 * i]), hi = __uint_as_float(r0[2 * i + 1]);
                        float lo1 = __uint_as_float(r1[2 * i]), hi1 = __uint_as_float(r1[2 * i + 1]);
                        if (KIND == 1) {
                            lo = __fmul_rn(lo, alpha);
                            hi = __fmul_rn(hi, alpha);
                            lo1 = __fmul_rn(lo1, alpha);
                            hi1 = __fmul_rn(hi1, alpha);
                        }
                        const __nv_bfloat162 b0 = __floats2bfloat162_rn(lo, hi);
                        const __nv_bfloat162 b1 = __floats2bfloat162_rn(lo1, hi1);
                        packed[c * 16 + i] = *reinterpret_cast<const uint32_t*>(&b0);
                        packed[c * 16 + 16 + i] = *reinterpret_cast<const uint32_t*>(&b1);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acce_leader);
                if (p.tma_store) {
                    // 64 columns at a time: rows into the warp's 128B-swizzled staging tile, then one
                    // TMA store (clipped at the M / N edges), so the output leaves in full lines
                    uint8_t* stg = smem + C::OFF_STG + (warp - 2) * C::STG_BYTES;
#pragma unroll
                    for (int h = 0; h < COLS / 64; ++h) {
                        if (lane == 0) bulk_wait_group_read0();
                        __syncwarp();
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            *reinterpret_cast<uint4*>(stg + lane * 128 + ((c ^ (lane & 7)) * 16)) =
                                make_uint4(packed[h * 32 + 4 * c], packed[h * 32 + 4 * c + 1], packed[h * 32 + 4 * c + 2],
                                           packed[h * 32 + 4 * c + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        const int ys = mt * 256 + static_cast<int>(rank) * 128 + sub * 32;
                        if (lane == 0 && ys < p.M && n0 + h * 64 < p.N) {  // boxes wholly past the edge are skipped
                            tma_store_2d(&tma_out, stg, n0 + h * 64, ys);
                            bulk_commit_group();
                        }
                    }
                } else if (m < p.M) {
                    if (vec) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + n0);
#pragma unroll
                        for (int v = 0; v < COLS / 8; ++v)
                            dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
                    } else {
                        uint16_t* o16 = reinterpret_cast<uint16_t*>(orow);
#pragma unroll
                        for (int v = 0; v < COLS / 2; ++v) {
                            const int n = n0 + 2 * v;
                            if (n < p.N) o16[n] = static_cast<uint16_t>(packed[v] & 0xFFFFu);
                            if (n + 1 < p.N) o16[n + 1] = static_cast<uint16_t>(packed[v] >> 16);
                        }
                    }
                }
            } else {
                float* orow = static_cast<float*>(p.out) + static_cast<int64_t>(m) * p.N;
                const bool vec = (p.N & 3) == 0;
#pragma unroll 1
                for (int c = 0; c < COLS / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(t_row + c * 32, r);
                    tmem_ld_wait();
                    if (m < p.M) {
                        const int nb = n0 + c * 32;
                        if (vec && nb + 32 <= p.N) {
                            float4* dst = reinterpret_cast<float4*>(orow + nb);
#pragma unroll
                            for (int v = 0; v < 8; ++v) {
                                float4 f;
                                f.x = __fmul_rn(__uint_as_float(r[4 * v]), alpha);
                                f.y = __fmul_rn(__uint_as_float(r[4 * v + 1]), alpha);
                                f.z = __fmul_rn(__uint_as_float(r[4 * v + 2]), alpha);
                                f.w = __fmul_rn(__uint_as_float(r[4 * v + 3]), alpha);
                                dst[v] = f;
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (nb + i < p.N) orow[nb + i] = __fmul_rn(__uint_as_float(r[i]), alpha);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acce_leader);
            }
            if (++acc == C::ACC) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    if (warp >= 2 && lane == 0) bulk_wait_group0();  // output stores of this warp have landed
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no CTA leaves while its peer may still signal its barriers or use its TMEM
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host side

// 2-D byte tensor [rows][row_bytes], box of 128 bytes x box_rows, 128-byte swizzle, zero fill.
bool make_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_rows) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {row_bytes, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KIND, int BN, int STAGES, bool F32>
int run(const void* A_q, const void* B_q, GemmArgs args, cudaStream_t stream, bool pdl) {
    using C = Cfg<KIND, BN, STAGES>;
    auto kern = gemm_kernel<KIND, BN, STAGES, F32>;
    const int row_bytes = args.K / C::EPB;
    CUtensorMap ta, tb;
    if (!make_map(&ta, A_q, row_bytes, args.M, kBM) || !make_map(&tb, B_q, row_bytes, args.N, BN)) return MXQ_ERR_CUDA;
    args.m_tiles = static_cast<int>(ceil_div(args.M, kBM));
    args.n_tiles = static_cast<int>(ceil_div(args.N, BN));
    args.k_stages = static_cast<int>(ceil_div(args.K, C::BK));
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
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, args) != cudaSuccess) return MXQ_ERR_CUDA;
    return MXQ_OK;
}

// bf16 output [M][N] for TMA stores: boxes of 32 rows x 64 columns (128 bytes), 128B swizzle.
bool make_out_map(CUtensorMap* m, void* base, int64_t M, int64_t N) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
    cuuint32_t box[2] = {64, 32};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// Swizzled scales as rows of 256 bytes (two per 512-byte tile); a box covers `tiles` tiles.
bool make_sf_map(CUtensorMap* m, const void* base, int64_t rows, int64_t kblocks, uint32_t tiles) {
    auto enc = encode_fn();
    if (!enc) return false;
    const uint64_t half_rows = static_cast<uint64_t>(swizzled_sf_bytes(rows, kblocks) / 256);
    cuuint64_t dims[2] = {256, half_rows};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {256, 2 * tiles};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KIND, int STAGES, int BN, bool F32>
int run_pair(const void* A_q, const void* B_q, GemmArgs args, cudaStream_t stream, bool pdl) {
    using C = PairCfg<KIND, STAGES, BN>;
    auto kern = gemm_pair_kernel<KIND, STAGES, BN, F32>;
    const int row_bytes = args.K / C::EPB;
    const int64_t kblocks = args.K / C::BS;
    CUtensorMap ta, tb, tsa, tsb, to;
    if (!make_map(&ta, A_q, row_bytes, args.M, 128) || !make_map(&tb, B_q, row_bytes, args.N, C::B_ROWS) ||
        !make_sf_map(&tsa, args.a_sf, args.M, kblocks, C::SF_ATOMS) ||
        !make_sf_map(&tsb, args.b_sf, args.N, kblocks, C::SF_ATOMS))
        return MXQ_ERR_CUDA;
    memset(&to, 0, sizeof(to));
    args.tma_store = 0;
    if (!F32 && args.N % 8 == 0) {
        if (!make_out_map(&to, args.out, args.M, args.N)) return MXQ_ERR_CUDA;
        args.tma_store = 1;
    }
    args.m_tiles = static_cast<int>(ceil_div(args.M, 256));
    args.n_tiles = static_cast<int>(ceil_div(args.N, BN));
    // raster groups of M tiles whose A codes and scales fit in about 24 MB, so that A stays in L2
    // while B streams past it; where the whole of A fits, the plain M-fastest order (measured on
    // NVFP4 8192 x 5120 x 17408, 71 MB of A codes: 296 -> 275 us with groups of 8-16; groups only
    // slowed the shapes whose A fits)
    const int64_t a_tile_bytes = 256 * (static_cast<int64_t>(args.K) / C::EPB + args.K / C::BS);
    const int64_t group = (int64_t{24} << 20) / a_tile_bytes;
    args.group_m = group < 1 ? 1 : (group < args.m_tiles ? static_cast<int>(group) : args.m_tiles);
    args.k_stages = static_cast<int>(ceil_div(args.K, C::BK));
    int dev = 0;
    cudaGetDevice(&dev);
    static bool attr_done[64] = {};
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
            return MXQ_ERR_CUDA;
        attr_done[dev] = true;
    }
    const int64_t tiles = static_cast<int64_t>(args.m_tiles) * args.n_tiles;
    const int64_t max_pairs = sm_count() / 2;
    const int pairs = static_cast<int>(tiles < max_pairs ? tiles : max_pairs);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, tsa, tsb, to, args) != cudaSuccess) return MXQ_ERR_CUDA;
    return MXQ_OK;
}

template <int KIND, bool F32>
int run_splitk(const void* A_q, const void* B_q, GemmArgs args, int splits, cudaStream_t stream, bool pdl) {
    using C = Cfg<KIND, 128, 6>;
    auto kern = gemm_splitk_kernel<KIND, F32>;
    const int row_bytes = args.K / C::EPB;
    CUtensorMap ta, tb;
    const uint32_t a_rows = static_cast<uint32_t>(ceil_div(args.M, 8) * 8);
    if (!make_map(&tb, B_q, row_bytes, args.N, 128) || !make_map(&ta, A_q, row_bytes, args.M, a_rows))
        return MXQ_ERR_CUDA;
    args.a_box_bytes = a_rows * 128;
    args.m_tiles = 1;
    args.n_tiles = static_cast<int>(ceil_div(args.N, 128));
    args.k_stages = static_cast<int>(ceil_div(args.K, C::BK));
    args.k_split = static_cast<uint32_t>(splits);
    int dev = 0;
    cudaGetDevice(&dev);
    static bool attr_done[64] = {};
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
            return MXQ_ERR_CUDA;
        attr_done[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(args.n_tiles * splits);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, args) != cudaSuccess) return MXQ_ERR_CUDA;
    return MXQ_OK;
}

// bf16 out [M][N] in boxes of 128 columns x 32 rows, no swizzle (the few-token kernel's output
// tile); TMA stores clip at the M and N edges.  Needs N % 8 == 0.
bool make_out_tok_map(CUtensorMap* m, void* base, int64_t M, int64_t N) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
    cuuint32_t box[2] = {128, 32};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int KIND, int WG, bool F32, int QRULE>
int run_decode(const void* x, const void* B_q, GemmArgs args, int splits, cudaStream_t stream) {
    using C = DecCfg<KIND, WG>;
    auto kern = gemm_decode_kernel<KIND, WG, F32, QRULE>;
    CUtensorMap tx, tw, to;
    // x: bf16 rows of 2 K bytes in boxes of 128 bytes (64 elements) x 32 rows; W codes 128 WG rows x 128 bytes
    if (!make_map(&tx, x, 2 * static_cast<uint64_t>(args.K), args.M, C::TOK) ||
        !make_map(&tw, B_q, args.K / C::EPB, args.N, 128 * WG))
        return MXQ_ERR_CUDA;
    memset(&to, 0, sizeof(to));
    args.tma_store = 0;
    if (!F32 && args.N % 8 == 0) {
        if (!make_out_tok_map(&to, args.out, args.M, args.N)) return MXQ_ERR_CUDA;
        args.tma_store = 1;
    }
    args.m_tiles = 1;
    args.n_tiles = static_cast<int>(ceil_div(args.N, 128 * WG));
    args.k_stages = static_cast<int>(ceil_div(args.K, C::BK));
    args.k_split = static_cast<uint32_t>(splits);
    if (WG > 1 && splits != 1) return MXQ_ERR_UNSUPPORTED;  // two weight groups are never split along K
    int dev = 0;
    cudaGetDevice(&dev);
    static bool attr_done[64] = {};
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
            return MXQ_ERR_CUDA;
        attr_done[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(args.n_tiles * splits);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, tx, tw, to, args) != cudaSuccess) return MXQ_ERR_CUDA;
    return MXQ_OK;
}

// bf16 out [M][N] in boxes of 32 columns (64 bytes) x 32 rows, 64B swizzle (16-byte piece q of row
// r at piece q ^ ((r >> 1) & 3)); TMA stores clip at the M and N edges.  Needs N % 8 == 0.
bool make_out32_map(CUtensorMap* m, void* base, int64_t M, int64_t N) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int KIND, bool F32, int QRULE>
int run_rowq(const void* x, const void* B_q, GemmArgs args, int splits, cudaStream_t stream) {
    using C = RowqCfg<KIND>;
    auto kern = gemm_rowq_kernel<KIND, F32, QRULE>;
    CUtensorMap tx, tb, to;
    // x: bf16 rows of 2 K bytes in boxes of 128 bytes (64 elements) x 128 rows; W codes as the GEMM's
    if (!make_map(&tx, x, 2 * static_cast<uint64_t>(args.K), args.M, 128) ||
        !make_map(&tb, B_q, args.K / C::EPB, args.N, 128))
        return MXQ_ERR_CUDA;
    memset(&to, 0, sizeof(to));
    args.tma_store = 0;
    if (!F32 && args.N % 8 == 0) {
        if (!make_out32_map(&to, args.out, args.M, args.N)) return MXQ_ERR_CUDA;
        args.tma_store = 1;
    }
    args.m_tiles = static_cast<int>(ceil_div(args.M, 128));
    args.n_tiles = 1;
    args.k_stages = static_cast<int>(ceil_div(args.K, C::BK));
    args.k_split = static_cast<uint32_t>(splits);
    int dev = 0;
    cudaGetDevice(&dev);
    static bool attr_done[64] = {};
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
            return MXQ_ERR_CUDA;
        attr_done[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(args.m_tiles * splits);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, tx, tb, to, args) != cudaSuccess) return MXQ_ERR_CUDA;
    return MXQ_OK;
}

// K splits of the small-N kernel: as many as keep all M tiles' clusters resident at once (at most
// 4), each split owning at least one K stage.
int rowq_splits(int64_t M, int64_t K, int bk) {
    const int64_t m_tiles = ceil_div(M, 128);
    const int64_t k_stages = ceil_div(K, bk);
    int64_t s = sm_count() / m_tiles;
    if (s > static_cast<int64_t>(kMaxSplits)) s = kMaxSplits;
    if (s > k_stages) s = k_stages;
    if (s < 2) return 1;
    const int64_t per = ceil_div(k_stages, s);
    return static_cast<int>(ceil_div(k_stages, per));
}

// K splits for a one-row-tile problem: as many as keep every cluster of the grid resident at once
// (at most 4), each split owning at least one K stage.
int splitk_count(int64_t N, int64_t K, int bk) {
    const int64_t n_tiles = ceil_div(N, 128);
    const int64_t k_stages = ceil_div(K, bk);
    int64_t s = sm_count() / n_tiles;
    if (s > static_cast<int64_t>(kMaxSplits)) s = kMaxSplits;
    if (s > k_stages) s = k_stages;
    if (s < 2) return 1;
    const int64_t per = ceil_div(k_stages, s);
    return static_cast<int>(ceil_div(k_stages, per));
}

template <int KIND, bool F32>
int dispatch_bn(const void* A_q, const void* B_q, const GemmArgs& args, cudaStream_t stream, bool pdl) {
    // More than 128 rows: CTA pairs on 256 x 256 tiles with one accumulator.  Up to 128 rows
    // (decode): one CTA per 128 x 128 tile, which gives the most CTAs for the weight stream.
    // 256 x 192 tiles with two accumulators (BN = 192) remove the drain bubble at tile boundaries
    // but measured slower on the prefill problems.
    if (args.M > 128) return run_pair<KIND, 5, 256, F32>(A_q, B_q, args, stream, pdl);
    const int splits = splitk_count(args.N, args.K, Cfg<KIND, 128, 6>::BK);
    if (splits > 1) return run_splitk<KIND, F32>(A_q, B_q, args, splits, stream, pdl);
    // more 128-wide tiles than SMs: 128 x 256 tiles halve the tile count (one tile per CTA up to
    // N = 256 x SMs) and read the A rows once per 256 weight rows
    if (ceil_div(args.N, 128) > sm_count()) return run<KIND, 256, 4, F32>(A_q, B_q, args, stream, pdl);
    return run<KIND, 128, 6, F32>(A_q, B_q, args, stream, pdl);
}

}  // namespace

int launch_gemm(const void* A_q, const uint8_t* A_sf, const void* B_q, const uint8_t* B_sf, const float* g_A,
                const float* g_B, int64_t M, int64_t N, int64_t K, int fmt, int out_type, void* out,
                cudaStream_t stream, bool pdl_secondary) {
    GemmArgs a = {};
    a.a_sf = A_sf;
    a.b_sf = B_sf;
    a.g_a = g_A;
    a.g_b = g_B;
    a.out = out;
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.sf_col_tiles = static_cast<int>(ceil_div(K / block_size(fmt), 4));
    a.b_row_tiles = static_cast<int>(ceil_div(N, 128));
    a.status = status_ptr();
    const bool f32 = out_type == MXQ_OUT_FP32;
    switch (fmt) {
        case MXQ_MXFP4:
            return f32 ? dispatch_bn<0, true>(A_q, B_q, a, stream, pdl_secondary)
                       : dispatch_bn<0, false>(A_q, B_q, a, stream, pdl_secondary);
        case MXQ_NVFP4:
            return f32 ? dispatch_bn<1, true>(A_q, B_q, a, stream, pdl_secondary)
                       : dispatch_bn<1, false>(A_q, B_q, a, stream, pdl_secondary);
        default:
            return f32 ? dispatch_bn<2, true>(A_q, B_q, a, stream, pdl_secondary)
                       : dispatch_bn<2, false>(A_q, B_q, a, stream, pdl_secondary);
    }
}

namespace {
template <int KIND, bool F32>
int fused_rule(const void* W_q, const GemmArgs& a, int rule, int splits, cudaStream_t stream) {
    if (splits >= 2)  // 128 weight rows per CTA, K split over a cluster
        return rule == MXQ_RULE_CEIL ? run_decode<KIND, 1, F32, MXQ_RULE_CEIL>(a.x, W_q, a, splits, stream)
                                     : run_decode<KIND, 1, F32, MXQ_RULE_EVEN>(a.x, W_q, a, splits, stream);
    // many weight rows: 256 per CTA, no K split
    return rule == MXQ_RULE_CEIL ? run_decode<KIND, 2, F32, MXQ_RULE_CEIL>(a.x, W_q, a, 1, stream)
                                 : run_decode<KIND, 2, F32, MXQ_RULE_EVEN>(a.x, W_q, a, 1, stream);
}
template <int KIND, bool F32>
int rowq_rule(const void* x, const void* W_q, const GemmArgs& a, int rule, int splits, cudaStream_t stream) {
    return rule == MXQ_RULE_CEIL ? run_rowq<KIND, F32, MXQ_RULE_CEIL>(x, W_q, a, splits, stream)
                                 : run_rowq<KIND, F32, MXQ_RULE_EVEN>(x, W_q, a, splits, stream);
}

// Few output columns and more tokens than the few-token kernel quantizes itself: one column tile, so
// the small-N kernel reads each activation row once and quantizes it on the way in.
bool rowq_applies(int64_t M, int64_t N) { return M > 32 && N <= RowqCfg<0>::BN; }
}  // namespace

int linear_fused_splits(int64_t M, int64_t N, int64_t K, int fmt) {
    if (rowq_applies(M, N)) return rowq_splits(M, K, fmt == MXQ_MXFP8 ? RowqCfg<2>::BK : RowqCfg<0>::BK);
    // up to 32 tokens: the few-token kernel, with 128 weight rows per CTA and a K split where that
    // fills the SMs, else with 256 weight rows per CTA where those tiles fit one wave; with more
    // weight rows than that, the quantizer and the persistent GEMM
    if (M > 32) return 0;
    const int bk = fmt == MXQ_MXFP8 ? Cfg<2, 128, 6>::BK : Cfg<0, 128, 6>::BK;
    const int splits = splitk_count(N, K, bk);
    if (splits >= 2) return splits;
    return ceil_div(N, 256) <= sm_count() ? 1 : 0;
}

int launch_linear_fused(const void* x, const void* W_q, const uint8_t* W_sf, const float* g_W, const float* g_A,
                        int64_t M, int64_t N, int64_t K, int fmt, int rule, int out_type, void* out,
                        cudaStream_t stream) {
    const int splits = linear_fused_splits(M, N, K, fmt);
    const bool rowq = rowq_applies(M, N);
    if (!rowq && splits < 1) return kNotFused;
    GemmArgs a = {};
    a.x = x;
    a.b_sf = W_sf;
    a.g_a = g_A;
    a.g_b = g_W;
    a.out = out;
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.sf_col_tiles = static_cast<int>(ceil_div(K / block_size(fmt), 4));
    a.b_row_tiles = static_cast<int>(ceil_div(N, 128));
    a.status = status_ptr();
    const bool f32 = out_type == MXQ_OUT_FP32;
    if (rowq) {
        switch (fmt) {
            case MXQ_MXFP4:
                return f32 ? rowq_rule<0, true>(x, W_q, a, rule, splits, stream)
                           : rowq_rule<0, false>(x, W_q, a, rule, splits, stream);
            case MXQ_NVFP4:
                return f32 ? run_rowq<1, true, 0>(x, W_q, a, splits, stream) : run_rowq<1, false, 0>(x, W_q, a, splits, stream);
            default:
                return f32 ? rowq_rule<2, true>(x, W_q, a, rule, splits, stream)
                           : rowq_rule<2, false>(x, W_q, a, rule, splits, stream);
        }
    }
    switch (fmt) {
        case MXQ_MXFP4:
            return f32 ? fused_rule<0, true>(W_q, a, rule, splits, stream) : fused_rule<0, false>(W_q, a, rule, splits, stream);
        case MXQ_NVFP4:
            return f32 ? fused_rule<1, true>(W_q, a, rule, splits, stream) : fused_rule<1, false>(W_q, a, rule, splits, stream);
        default:
            return f32 ? fused_rule<2, true>(W_q, a, rule, splits, stream) : fused_rule<2, false>(W_q, a, rule, splits, stream);
    }
}

}  // namespace mxq
