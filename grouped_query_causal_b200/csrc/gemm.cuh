// gemm.cuh -- the projections around the attention: y = x W^T on the 5th-generation
// tensor cores (sm_100a).
//
// The "Qwen3" walkthrough's attention forward starts with the fused projection
// qkv = qkv_proj(hidden_states) (steps 1-3: split into q, k, v and viewed per head) and
// ends with output = o_proj(o.flatten(1, -1)) (step 7); "Qwen3系列1-理论基础&真实结构"
// D1-2 gives a linear layer as Y = XW + b with no b for Qwen3's projections, and D1-4
// (Q4/Q5) the concatenation of the heads followed by W_O.  Both are one dense
// contraction, y[m][n] = sum_k x[m][k] w[n][k] with x [M, K] and w [N, K] bf16 (both
// K-major, nn.Linear's layout), accumulated in fp32 and stored as bf16 or fp32.
//
// gemm_kernel: persistent, one CTA per SM walking 128 x 256 output tiles (grouped by 8
// M-blocks so that neighbouring CTAs share W tiles in L2).  Warp 0 streams 128 x 64 x-
// tiles and 256 x 64 w-tiles into a 4-stage ring with TMA (128-byte swizzle); warp 1
// issues tcgen05.mma (M = 128, N = 256, K = 16; four per stage) into one of two TMEM
// accumulators of 256 fp32 columns; warps 4-7 drain the other accumulator (one output
// row per thread) to global memory while the next tile accumulates.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace gqa {

constexpr int kGemmBM = 128, kGemmBN = 256, kGemmBK = 64;
constexpr int kGemmStages = 4;
constexpr int kGemmGroupM = 8;
constexpr uint32_t kGemmABytes = kGemmBM * kGemmBK * 2;   // 16 KB
constexpr uint32_t kGemmBBytes = kGemmBN * kGemmBK * 2;   // 32 KB
constexpr uint32_t kGemmStageBytes = kGemmABytes + kGemmBBytes;
constexpr uint32_t kGemmOffStage = kGemmStages * kGemmStageBytes;   // epilogue staging: 4 warps x 32 rows x 128 B
constexpr uint32_t kGemmOffBar = kGemmOffStage + 4 * 32 * 128;
enum {
    GB_FULL = 0,                          // [stages] TMA -> MMA
    GB_EMPTY = kGemmStages,               // [stages] MMA (commit) -> TMA
    GB_ACC_FULL = 2 * kGemmStages,        // [2] MMA (commit) -> epilogue
    GB_ACC_EMPTY = 2 * kGemmStages + 2,   // [2] epilogue (128 arrivals) -> MMA
    GB_DRAIN = 2 * kGemmStages + 4,
    GB_NUM = 2 * kGemmStages + 5
};
constexpr uint32_t kGemmOffTmem = kGemmOffBar + GB_NUM * 8;
constexpr uint32_t kGemmSmemBytes = kGemmOffTmem + 16 + 1024;
constexpr int kGemmThreads = 256;   // warp 0 TMA, warp 1 MMA, warps 4-7 epilogue
static_assert(kGemmSmemBytes <= 232448, "shared memory budget");

struct GemmParams {
    void *y;            // [M, N] bf16 or fp32, row-major (row stride ldy elements)
    unsigned *err;
    int M, N, K;
    long long ldy;
    int y_fp32;         // 1: fp32 output, 0: bf16
    int mblocks, nblocks, ntiles;
};

// Tile t -> (m block, n block), grouped: kGemmGroupM consecutive M blocks share each n.
__device__ __forceinline__ void gemm_tile(const GemmParams &p, int t, int &mb, int &nb) {
    const int per_group = kGemmGroupM * p.nblocks;
    const int grp = t / per_group;
    const int first_m = grp * kGemmGroupM;
    const int gm = min(kGemmGroupM, p.mblocks - first_m);
    const int in = t % per_group;
    mb = first_m + in % gm;
    nb = in / gm;
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw_base & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    const uint32_t sbase = raw_base + pad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t bar0 = sbase + kGemmOffBar;
#define GBAR(i) (bar0 + 8u * static_cast<uint32_t>(i))

    if (tid == 0) {
        for (int i = 0; i < kGemmStages; ++i) {
            mbar_init(GBAR(GB_FULL + i), 1);
            mbar_init(GBAR(GB_EMPTY + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(GBAR(GB_ACC_FULL + i), 1);
            mbar_init(GBAR(GB_ACC_EMPTY + i), 128);
        }
        mbar_init(GBAR(GB_DRAIN), 1);
        fence_mbarrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_x);
        prefetch_tensormap(&tm_w);
    }
    if (warp == 1) {
        tmem_alloc(sbase + kGemmOffTmem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + kGemmOffTmem);
    const int ksteps = (p.K + kGemmBK - 1) / kGemmBK;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x) {
                int mb, nb;
                gemm_tile(p, t, mb, nb);
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const uint32_t st = it % kGemmStages, use = it / kGemmStages;
                    if (use > 0 && !mbar_wait(GBAR(GB_EMPTY + st), (use - 1) & 1, p.err)) {
                        ok = false;
                        break;
                    }
                    const uint32_t dst = sbase + st * kGemmStageBytes;
                    mbar_arrive_expect_tx(GBAR(GB_FULL + st), kGemmStageBytes);
                    tma_load_2d(dst, &tm_x, ks * kGemmBK, mb * kGemmBM, GBAR(GB_FULL + st));
                    tma_load_2d(dst + kGemmABytes, &tm_w, ks * kGemmBK, nb * kGemmBN, GBAR(GB_FULL + st));
                }
            }
            if (!ok) {
                // let the copies in flight land: the last armed phase of every stage
                for (uint32_t i = (it > kGemmStages ? it - kGemmStages : 0); i < it; ++i)
                    mbar_wait(GBAR(GB_FULL + i % kGemmStages), (i / kGemmStages) & 1, p.err);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kGemmBM, kGemmBN, false);
            uint32_t it = 0, acc_uses[2] = {0u, 0u};
            bool ok = true;
            int local = 0;
            for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x, ++local) {
                const int a = local & 1;
                // the epilogue must have drained this accumulator's previous tile
                if (acc_uses[a] > 0 && !mbar_wait_hint(GBAR(GB_ACC_EMPTY + a), (acc_uses[a] - 1) & 1, 20u, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(a) * kGemmBN;
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const uint32_t st = it % kGemmStages;
                    if (!mbar_wait_hint(GBAR(GB_FULL + st), (it / kGemmStages) & 1, 20u, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = sbase + st * kGemmStageBytes, sb = sa + kGemmABytes;
#pragma unroll
                    for (int kk = 0; kk < kGemmBK / 16; ++kk)
                        umma_bf16_ss(d, sw128_desc(sa + 32u * kk, 16, 1024), sw128_desc(sb + 32u * kk, 16, 1024), idesc,
                                     (ks > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(GBAR(GB_EMPTY + st));
                }
                if (!ok) break;
                umma_commit(GBAR(GB_ACC_FULL + a));
                ++acc_uses[a];
            }
            umma_commit(GBAR(GB_DRAIN));
            mbar_wait(GBAR(GB_DRAIN), 0, p.err);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                 // TMEM lanes 32 q .. 32 q + 31
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        uint32_t acc_uses[2] = {0u, 0u};
        int local = 0;
        for (int t = blockIdx.x; t < p.ntiles; t += gridDim.x, ++local) {
            const int a = local & 1;
            int mb, nb;
            gemm_tile(p, t, mb, nb);
            if (!__all_sync(0xffffffffu, mbar_wait(GBAR(GB_ACC_FULL + a), acc_uses[a] & 1, p.err))) break;
            ++acc_uses[a];
            tc_fence_after();
            const int row0 = mb * kGemmBM + q * 32;   // this warp's 32 output rows
            const int col0 = nb * kGemmBN;
            const uint32_t tacc = tmem + lane_base + static_cast<uint32_t>(a) * kGemmBN;
            // Each 32-column chunk: every thread stages its row (16-byte granules swizzled by
            // row, so that no two lanes of a quarter-warp hit the same banks), then the warp
            // copies its 32 rows out whole-row: 4 fp32 rows (128 B each) or 8 bf16 rows (64 B
            // each) per instruction instead of 32 scattered 16-byte pieces.
            const uint32_t stg = sbase + kGemmOffStage + static_cast<uint32_t>(q) * 32 * 128;
#pragma unroll 1
            for (int c = 0; c < kGemmBN / 32; ++c) {
                float v[32];
                tmem_ld32(tacc + 32 * c, v);
                tmem_wait_ld();
                const int col = col0 + 32 * c;
                if (p.y_fp32) {
#pragma unroll
                    for (int g = 0; g < 8; ++g)
                        st_shared_v4(stg + lane * 128 + ((g ^ (lane & 7)) << 4),
                                     make_uint4(__float_as_uint(v[4 * g]), __float_as_uint(v[4 * g + 1]),
                                                __float_as_uint(v[4 * g + 2]), __float_as_uint(v[4 * g + 3])));
                    __syncwarp();
                    const int g = lane & 7;
#pragma unroll
                    for (int it = 0; it < 8; ++it) {
                        const int r = it * 4 + (lane >> 3);
                        const uint4 u = ld_shared_v4(stg + r * 128 + ((g ^ (r & 7)) << 4));
                        if (row0 + r < p.M && col < p.N)   // N is a multiple of 32
                            *reinterpret_cast<uint4 *>(static_cast<float *>(p.y) + (row0 + r) * p.ldy + col + 4 * g) = u;
                    }
                } else {
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        st_shared_v4(stg + lane * 128 + ((g ^ (lane & 7)) << 4),
                                     make_uint4(pack_bf16x2(v[8 * g], v[8 * g + 1]), pack_bf16x2(v[8 * g + 2], v[8 * g + 3]),
                                                pack_bf16x2(v[8 * g + 4], v[8 * g + 5]),
                                                pack_bf16x2(v[8 * g + 6], v[8 * g + 7])));
                    __syncwarp();
                    const int g = lane & 3;
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int r = it * 8 + (lane >> 2);
                        const uint4 u = ld_shared_v4(stg + r * 128 + ((g ^ (r & 7)) << 4));
                        if (row0 + r < p.M && col < p.N)
                            *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.y) + (row0 + r) * p.ldy + col + 8 * g) = u;
                    }
                }
                __syncwarp();   // the warp's staging rows are free again
            }
            tc_fence_before();
            mbar_arrive(GBAR(GB_ACC_EMPTY + a));
        }
        tc_fence_before();
    }
#undef GBAR
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace gqa
