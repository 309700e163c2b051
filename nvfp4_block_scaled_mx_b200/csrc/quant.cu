// quant.cu -- bf16 -> MXFP4 (EVEN / CEIL), NVFP4 and MXFP8 block quantizer, scale swizzle,
// NVFP4 global scale, and the bounded-wait self-test kernel.
//
// The quantizer is a single streaming pass over x.  x is read as rows of 64 bytes (32 elements:
// one MX block or two NVFP4 blocks) by TMA, 256 rows per box, into a 2-stage shared-memory ring
// with a 64-byte swizzle (5 CTAs per SM); each thread then owns two 32-element rows of a box (their
// four 16-byte pieces sit in different banks), takes the block amax on the bf16 bit patterns,
// derives the scale, and writes 16 (FP4) or 32 (FP8) bytes of packed codes per row plus the scale
// bytes, either row-major or directly in the swizzled tensor-core layout (4 blocks' bytes gathered
// across lanes into one 32-bit store where a row's block count allows).  Fake quantization runs the
// same ring and decodes the codes back to bf16 in place.
#include <cstring>

#include "dequant.cuh"
#include "mxq_device.cuh"
#include "mxq_internal.h"
#include "quant_block.cuh"

namespace mxq {
namespace {


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


// Scale byte offset of block `blk` (row-major block index) in the requested layout.
template <bool SWZ>
__device__ __forceinline__ uint32_t scale_offset(uint32_t blk, uint32_t kblocks, uint64_t kb_magic, uint32_t col_tiles) {
    if constexpr (!SWZ) return blk;
    const uint32_t row = div_magic(blk, kblocks, kb_magic);
    const uint32_t kc = blk - row * kblocks;
    return swz_offset(row, kc, col_tiles);
}

// Quantize one 32-element row w (16 bf16x2 words) with unit index u: one MX block (MXFP4 / MXFP8)
// or two NVFP4 blocks.  Codes: 16 bytes (FP4) or 32 bytes (FP8), coalesced across the warp.  Every
// lane of the warp calls this (rows past the end hold the TMA's zero fill; `valid` masks their
// stores), so that the scale bytes can be gathered across lanes: when a row's block count is a
// multiple of 4 (pack_sf), the 4 scale bytes of 4 consecutive blocks sit in one aligned 32-bit word
// of either layout, and lane 4j (MX) or 2j (NVFP4, two blocks per unit) stores that word for
// itself and its neighbours; otherwise each block's byte is stored on its own.
template <int FMT, int RULE, bool SWZ, bool OBS>
__device__ __forceinline__ void quantize_unit(const uint32_t (&w)[16], int64_t u, bool valid, bool pack_sf, float g,
                                              const float* tab_d, const float* tab_r, uint32_t kblocks,
                                              uint64_t kb_magic, uint32_t col_tiles, uint8_t* __restrict__ q,
                                              uint8_t* __restrict__ sf, uint32_t& seen) {
    uint32_t codes[8];
    const uint32_t sc = quantize32<FMT, RULE, OBS>(w, g, tab_d, tab_r, codes, seen);
    if (valid) {
        if constexpr (FMT == MXQ_MXFP8) {
            uint4* dst = reinterpret_cast<uint4*>(q) + 2 * u;
            dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
            dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
        } else {
            reinterpret_cast<uint4*>(q)[u] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
        }
    }
    constexpr int BLOCKS = (FMT == MXQ_NVFP4) ? 2 : 1;  // scale bytes per unit
    const uint32_t blk = static_cast<uint32_t>(BLOCKS * u);
    if (pack_sf) {
        const uint32_t lane = threadIdx.x & 31u;
        uint32_t word;
        bool leader;
        if constexpr (BLOCKS == 2) {
            word = (sc & 0xFFFFu) | (__shfl_down_sync(0xFFFFFFFFu, sc, 1) << 16);
            leader = (lane & 1u) == 0;
        } else {
            word = (sc & 0xFFu) | ((__shfl_down_sync(0xFFFFFFFFu, sc, 1) & 0xFFu) << 8) |
                   ((__shfl_down_sync(0xFFFFFFFFu, sc, 2) & 0xFFu) << 16) | (__shfl_down_sync(0xFFFFFFFFu, sc, 3) << 24);
            leader = (lane & 3u) == 0;
        }
        // a leader's block index is a multiple of 4 and n_units * BLOCKS is too, so the word's
        // other blocks are valid whenever the leader's is
        if (leader && valid)
            *reinterpret_cast<uint32_t*>(sf + scale_offset<SWZ>(blk, kblocks, kb_magic, col_tiles)) = word;
    } else if (valid) {
#pragma unroll
        for (int b = 0; b < BLOCKS; ++b)
            sf[scale_offset<SWZ>(blk + b, kblocks, kb_magic, col_tiles)] = static_cast<uint8_t>(sc >> (8 * b));
    }
}

__device__ __forceinline__ float e4m3_decode(uint32_t c) {
    const float mag = e4m3_decode_pos(c & 0x7Fu);
    return (c & 0x80u) ? -mag : mag;
}

// 4 E4M3 codes times an arbitrary fp32 s, rounded as fl32(elem * s) and then to bf16.
__device__ __forceinline__ uint2 e4m3x4_fmul(uint32_t c, float s) {
    uint32_t o[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(__fmul_rn(e4m3_decode((c >> (16 * i)) & 0xFFu), s),
                                                       __fmul_rn(e4m3_decode((c >> (16 * i + 8)) & 0xFFu), s));
        o[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return make_uint2(o[0], o[1]);
}

// One 32-element unit fake-quantized: the codes and scales of quantize_unit (quantize32), decoded in
// the format's precision (MX: elem * 2^e, exact; NVFP4: fl(elem * d)) and rounded once to bf16;
// 64 bytes out.  MX decodes multiply in bf16 by a power of two where every product is a normal
// bf16 (scale codes [2, 128] for E2M1, [10, 134] for E4M3: exact, hence the same value), else in
// fp32.
template <int FMT, int RULE>
__device__ __forceinline__ void fake_unit(const uint32_t (&w)[16], float g, const float* tab_d, const float* tab_r,
                                          uint4 (&dst)[4]) {
    uint32_t codes[8], seen = 0;
    const uint32_t sc = quantize32<FMT, RULE, false>(w, g, tab_d, tab_r, codes, seen);
    if constexpr (FMT == MXQ_NVFP4) {
        const float d0 = tab_d[sc & 0xFFu], d1 = tab_d[sc >> 8];
        dst[0] = dequant8_fmul(codes[0], d0);
        dst[1] = dequant8_fmul(codes[1], d0);
        dst[2] = dequant8_fmul(codes[2], d1);
        dst[3] = dequant8_fmul(codes[3], d1);
    } else if constexpr (FMT == MXQ_MXFP4) {
        if (sc >= 2u && sc <= 128u) {
            const uint32_t f2 = mx_factor2(sc);
#pragma unroll
            for (int h = 0; h < 4; ++h) dst[h] = dequant8_mul(codes[h], f2);
        } else {
            const float s = pow2f(static_cast<int>(sc) - 127);
#pragma unroll
            for (int h = 0; h < 4; ++h) dst[h] = dequant8_cvt(codes[h], s);
        }
    } else {
        if (sc >= 10u && sc <= 134u) {
            const uint32_t f2 = mx8_factor2(sc);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const uint2 lo = e4m3x4_mul(codes[2 * h], f2), hi = e4m3x4_mul(codes[2 * h + 1], f2);
                dst[h] = make_uint4(lo.x, lo.y, hi.x, hi.y);
            }
        } else {
            const float s = pow2f(static_cast<int>(sc) - 127);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const uint2 lo = e4m3x4_fmul(codes[2 * h], s), hi = e4m3x4_fmul(codes[2 * h + 1], s);
                dst[h] = make_uint4(lo.x, lo.y, hi.x, hi.y);
            }
        }
    }
}

constexpr int kQuantStages = 2;
constexpr int kQuantRows = 256;                       // 64-byte rows (32 elements) per TMA box, two per thread
constexpr int kQuantBoxThreads = kQuantRows / 2;
constexpr int kQuantStageBytes = kQuantRows * 64;     // 16 KB of bf16 per stage
constexpr int kQuantCtasPerSm = 5;
// ring, barriers, NVFP4 per-code tables of d and 1/d, and 1024-byte alignment slack
constexpr int kQuantSmem = kQuantStages * kQuantStageBytes + kQuantStages * 8 + 2 * 128 * 4 + 1024;

// x streams through a 2-stage ring of TMA boxes (256 rows of 64 bytes, 64-byte swizzle) in each of
// up to 5 CTAs of 128 threads per SM; each CTA takes boxes blockIdx.x, blockIdx.x + gridDim.x, ...
// and each thread quantizes two rows of a box (two independent dependency chains).  One barrier
// per box: after it every thread has finished with the previous stage, which thread 0 then refills
// with the box kQuantStages - 1 ahead.
// OBS (NVFP4 only): gptr is a running amax; g = fl(amax / (6*448)) and the tensor amax of x is
// folded into *amax_out with one atomicMax per warp.
// FAKE: fake quantization instead: each thread writes its two bf16 output rows (64 bytes per unit)
// back over the input rows it read, and one TMA store per box (tmap_y, the same 64-byte swizzle)
// writes the box out whole, before the slot is refilled; sf is unused.
template <int FMT, int RULE, bool SWZ, bool OBS = false, bool FAKE = false>
__global__ void __launch_bounds__(kQuantBoxThreads, kQuantCtasPerSm)
    quantize_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_y,
                    int64_t n_units, uint32_t kblocks, uint64_t kb_magic,
                    uint32_t col_tiles, const float* __restrict__ gptr, uint8_t* __restrict__ q,
                    uint8_t* __restrict__ sf, unsigned int* __restrict__ amax_out, int* status,
                    const void* __restrict__ x_tail, bool tail, uint32_t rows) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(ring + kQuantStages * kQuantStageBytes);
    float* tab_d = reinterpret_cast<float*>(full + kQuantStages);
    float* tab_r = tab_d + 128;
    pdl_launch_dependents();
    const int64_t n_boxes = (n_units + kQuantRows - 1) / kQuantRows;
    const int64_t step = gridDim.x;
    if (threadIdx.x == 0) {
        if (n_boxes > 0) prefetch_tmap(&tmap_x);
        if (FAKE && n_boxes > 0) prefetch_tmap(&tmap_y);
        for (int st = 0; st < kQuantStages; ++st) mbar_init(&full[st], 1);
        fence_barrier_init();
    }
    // launched with programmatic serialization: everything above overlaps the previous kernel on
    // the stream; inputs are read and outputs written only after it has completed
    pdl_wait();
    if (threadIdx.x == 0) {
        const uint64_t pol = policy_evict_first();
        for (int st = 0; st < kQuantStages; ++st) {
            const int64_t b = blockIdx.x + st * step;
            if (b >= n_boxes) break;
            mbar_arrive_expect_tx(&full[st], kQuantStageBytes);
            tma_load_2d(&tmap_x, &full[st], ring + st * kQuantStageBytes, 0, static_cast<int>(b * kQuantRows), pol);
        }
    }
    if constexpr (SWZ && !FAKE) {
        // The swizzled layout's padding is zero: rows M .. (M rounded up to 128) of the last row
        // tile, and scale columns kblocks .. (kblocks rounded up to 4) of every row.  The main loop
        // never writes these bytes, so the grid zeroes them here, while the first boxes load.
        const uint32_t cols = col_tiles * 4u;
        const uint32_t pad_cols = cols - kblocks;
        const uint64_t n_row_pad = static_cast<uint64_t>(((rows + 127u) & ~127u) - rows) * cols;
        const uint64_t n_pad = n_row_pad + static_cast<uint64_t>(rows) * pad_cols;
        for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_pad;
             i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
            uint32_t r, c;
            if (i < n_row_pad) {
                r = rows + static_cast<uint32_t>(i / cols);
                c = static_cast<uint32_t>(i % cols);
            } else {
                const uint64_t j = i - n_row_pad;  // only reached when pad_cols > 0
                r = static_cast<uint32_t>(j / pad_cols);
                c = kblocks + static_cast<uint32_t>(j % pad_cols);
            }
            sf[swz_offset(r, c, col_tiles)] = 0;
        }
    }
    const float g = (FMT == MXQ_NVFP4) ? (OBS ? __fdiv_rn(*gptr, 2688.0f) : *gptr) : 1.0f;
    if constexpr (FMT == MXQ_NVFP4) nvfp4_tables(g, tab_d, tab_r);
    __syncthreads();
    uint32_t seen = 0;  // largest block amax (fp32 bits) this thread quantized, for OBS
    const bool pack_sf = (kblocks & 3u) == 0;
    // 64-byte swizzle: 16-byte piece c of row r sits at piece c ^ ((r >> 1) & 3); this thread takes
    // rows t and t + 128 of each box, which share the same swizzle
    const uint32_t my_row = smem_u32(ring) + threadIdx.x * 64u;
    const uint32_t sw = (threadIdx.x >> 1) & 3u;
    int it = 0;
    for (int64_t b = blockIdx.x; b < n_boxes; b += step, ++it) {
        const int st = it % kQuantStages;
        const bool ok = mbar_wait(&full[st], static_cast<uint32_t>(it / kQuantStages) & 1u, status, 30);
        // every thread is done with the previous stage and no thread leaves alone on a timeout
        if (__syncthreads_or(!ok)) break;
        if (threadIdx.x == 0 && it > 0) {
            const int prev = (it - 1) % kQuantStages;
            if constexpr (FAKE) {  // the previous box's output leaves before its slot is refilled
                tma_store_2d(&tmap_y, ring + prev * kQuantStageBytes, 0, static_cast<int>((b - step) * kQuantRows));
                bulk_commit_group();
                bulk_wait_group_read0();
            }
            const int64_t nb = b + (kQuantStages - 1) * step;
            if (nb < n_boxes) {
                mbar_arrive_expect_tx(&full[prev], kQuantStageBytes);
                tma_load_2d(&tmap_x, &full[prev], ring + prev * kQuantStageBytes, 0, static_cast<int>(nb * kQuantRows),
                            policy_evict_first());
            }
        }
        uint32_t w0[16], w1[16];
        const uint32_t row = my_row + static_cast<uint32_t>(st * kQuantStageBytes);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t piece = (static_cast<uint32_t>(i) ^ sw) << 4;
            const uint4 v0 = ld_shared_v4(row + piece);
            const uint4 v1 = ld_shared_v4(row + kQuantBoxThreads * 64 + piece);
            w0[4 * i + 0] = v0.x;
            w0[4 * i + 1] = v0.y;
            w0[4 * i + 2] = v0.z;
            w0[4 * i + 3] = v0.w;
            w1[4 * i + 0] = v1.x;
            w1[4 * i + 1] = v1.y;
            w1[4 * i + 2] = v1.z;
            w1[4 * i + 3] = v1.w;
        }
        const int64_t u = b * kQuantRows + threadIdx.x;
        if constexpr (FAKE) {
            uint4 o0[4], o1[4];
            fake_unit<FMT, RULE>(w0, g, tab_d, tab_r, o0);
            fake_unit<FMT, RULE>(w1, g, tab_d, tab_r, o1);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t piece = (static_cast<uint32_t>(i) ^ sw) << 4;
                st_shared_v4(row + piece, o0[i]);
                st_shared_v4(row + kQuantBoxThreads * 64 + piece, o1[i]);
            }
            fence_proxy_async_smem();  // read next by the TMA store
        } else {
            quantize_unit<FMT, RULE, SWZ, OBS>(w0, u, u < n_units, pack_sf, g, tab_d, tab_r, kblocks, kb_magic,
                                               col_tiles, q, sf, seen);
            quantize_unit<FMT, RULE, SWZ, OBS>(w1, u + kQuantBoxThreads, u + kQuantBoxThreads < n_units, pack_sf, g,
                                               tab_d, tab_r, kblocks, kb_magic, col_tiles, q, sf, seen);
        }
    }
    if constexpr (FAKE) {
        // the last box this CTA wrote (also after a timed-out wait, which ends the loop before the
        // store at the top of the next iteration)
        __syncthreads();
        if (threadIdx.x == 0 && it > 0) {
            tma_store_2d(&tmap_y, ring + ((it - 1) % kQuantStages) * kQuantStageBytes, 0,
                         static_cast<int>((blockIdx.x + static_cast<int64_t>(it - 1) * step) * kQuantRows));
            bulk_commit_group();
            bulk_wait_group0();
        }
    }
    if constexpr (FMT == MXQ_NVFP4) {
        // M * K = 16 (mod 32): the last NVFP4 block is half a 32-element row, quantized from global memory
        if (tail && blockIdx.x == 0 && threadIdx.x == 0) {
            const uint4* xt = reinterpret_cast<const uint4*>(x_tail);
            const uint4 v0 = xt[0], v1 = xt[1];
            const uint32_t wt[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            if constexpr (FAKE) {
                uint32_t codes[2];
                const uint32_t s = nvfp4_block<false>(wt, g, tab_d, tab_r, codes, seen);
                uint4* yt = reinterpret_cast<uint4*>(q) + n_units * 4;
                yt[0] = dequant8_fmul(codes[0], tab_d[s]);
                yt[1] = dequant8_fmul(codes[1], tab_d[s]);
            } else {
                uint32_t codes[2];
                const uint32_t s = nvfp4_block<OBS>(wt, g, tab_d, tab_r, codes, seen);
                reinterpret_cast<uint2*>(q)[2 * n_units] = make_uint2(codes[0], codes[1]);
                sf[scale_offset<SWZ>(static_cast<uint32_t>(2 * n_units), kblocks, kb_magic, col_tiles)] =
                    static_cast<uint8_t>(s);
            }
        }
    }
    if constexpr (OBS) {
        seen = __reduce_max_sync(0xFFFFFFFFu, seen);
        if ((threadIdx.x & 31) == 0 && seen != 0) atomicMax(amax_out, seen);
    }
}

// x [n_units][64 bytes] as a 2-D byte tensor, boxes of 256 rows, 64-byte swizzle.
bool make_x_map(CUtensorMap* m, const void* x, int64_t n_units) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(n_units)};
    cuuint64_t strides[1] = {64};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kQuantRows)};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(x), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT, int RULE, bool SWZ, bool OBS, bool FAKE = false>
cudaError_t launch_q_tma(const void* x, int64_t M, int64_t K, const float* g, void* q, void* sf, unsigned int* amax_out,
                         cudaStream_t stream) {
    const int64_t n_units = M * K / 32;
    const bool tail = (M * K) % 32 != 0;  // NVFP4 only: a last block of 16 elements
    const uint32_t kblocks = static_cast<uint32_t>(K / block_size(FMT));
    const uint32_t col_tiles = static_cast<uint32_t>(ceil_div(kblocks, 4));
    CUtensorMap tmap, tmap_y;
    memset(&tmap, 0, sizeof(tmap));
    memset(&tmap_y, 0, sizeof(tmap_y));
    if (n_units > 0 && !make_x_map(&tmap, x, n_units)) return cudaErrorInvalidValue;
    // fake quantization: the bf16 output has the input's layout, written box by box with TMA stores
    if (FAKE && n_units > 0 && !make_x_map(&tmap_y, q, n_units)) return cudaErrorInvalidValue;
    auto kern = quantize_kernel<FMT, RULE, SWZ, OBS, FAKE>;
    int dev = 0;
    cudaGetDevice(&dev);
    static bool attr_done[64] = {};
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kQuantSmem);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    int64_t blocks = ceil_div(n_units, static_cast<int64_t>(kQuantRows));
    const int64_t cap = static_cast<int64_t>(sm_count()) * kQuantCtasPerSm;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    // ceil(2^64 / kblocks); unused when kblocks == 1
    const uint64_t kb_magic =
        kblocks > 1 ? static_cast<uint64_t>(((static_cast<unsigned __int128>(1) << 64) + kblocks - 1) / kblocks) : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(kQuantBoxThreads);
    cfg.dynamicSmemBytes = kQuantSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmap, tmap_y, n_units, kblocks, kb_magic, col_tiles, g, static_cast<uint8_t*>(q),
                              static_cast<uint8_t*>(sf), amax_out, status_ptr(),
                              static_cast<const void*>(static_cast<const uint8_t*>(x) + n_units * 64), tail,
                              static_cast<uint32_t>(M));
}

template <int FMT, int RULE, bool SWZ>
cudaError_t launch_q(const void* x, int64_t M, int64_t K, const float* g, void* q, void* sf, cudaStream_t stream) {
    return launch_q_tma<FMT, RULE, SWZ, false>(x, M, K, g, q, sf, nullptr, stream);
}

// ------------------------------------------------------------------ fake quantization

template <int FMT, int RULE>
cudaError_t launch_fq(const void* x, int64_t M, int64_t K, const float* g, void* y, cudaStream_t stream) {
    // the quantizer's TMA-fed ring, writing bf16 (64 bytes per 32-element unit) instead of codes
    return launch_q_tma<FMT, RULE, false, false, true>(x, M, K, g, y, nullptr, nullptr, stream);
}

template <bool SWZ>
cudaError_t launch_q_running(const void* x, int64_t M, int64_t K, const float* amax_in, float* amax_out, void* q,
                             void* sf, cudaStream_t stream) {
    return launch_q_tma<MXQ_NVFP4, 0, SWZ, true>(x, M, K, amax_in, q, sf, reinterpret_cast<unsigned int*>(amax_out),
                                                 stream);
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
    if (layout == MXQ_SF_SWIZZLED) return launch_q_layout<true>(x, M, K, fmt, rule, g, q, sf, stream);
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
    if (layout == MXQ_SF_SWIZZLED) return launch_q_running<true>(x, M, K, amax_in, amax_out, q, sf, stream);
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
    if (e != cudaSuccess || g_out == nullptr) return e;  // mxq_amax stops at the tensor amax
    global_scale_finalize<<<1, 1, 0, stream>>>(amax_out, g_out);
    return cudaGetLastError();
}

cudaError_t launch_selftest_timeout(uint64_t timeout_ns, cudaStream_t stream) {
    selftest_timeout_kernel<<<1, 32, 0, stream>>>(status_ptr(), timeout_ns);
    return cudaGetLastError();
}

}  // namespace mxq
