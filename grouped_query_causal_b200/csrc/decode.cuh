// decode.cuh -- split-KV decode for sm_100a.
//
// One new query token per sequence attends to its whole KV cache ("Qwen3系列1-理论基础&
// 真实结构" D2-3: decode feeds a single token and is bound by reading the cache).  The
// work is bandwidth-bound: every cached K/V row is read exactly once, shared by the
// h = H/Hkv query heads of its group ("深入剖析Qwen3模型架构" 3.1.2).
//
//  decode_split_kernel: one CTA per (sequence, KV head, 1024-key chunk, head pass).
//    The h query vectors are normed + rotated at the query position in the prologue;
//    each warp streams 256 keys of the chunk with 16-byte loads (a half-warp per
//    256-byte key row, 16 rows per batch, the next batch's loads issued before the
//    current batch is used), first K (scores for all h heads), then V (weighted sum;
//    its first batch is requested before the softmax of the scores), with packed
//    two-lane fp32 FMAs (the kernel is otherwise issue-bound), and the four warp
//    partials are merged into one (m, l, O) per head.
//  decode_merge_kernel: log-sum-exp combination of the chunk partials of each
//    (sequence, query head):  O = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c.
//  decode_append_kernel: the decode step that first writes the new token into the
//    cache ("Qwen3系列1" D2-3: K and V enter the per-layer cache before attention):
//    k-hat = RoPE(RMSNorm(k_new; w_k)) at the token's position and v_new go to row
//    len of each sequence; the split kernel then attends to len + 1 rows.
#pragma once
#include <cuda_runtime.h>

#include "ptx.cuh"
#include "rope.cuh"

namespace gqa {

constexpr int kChunk = 1024;                // keys per split
constexpr int kWarpKeys = kChunk / 4;      // keys per warp
constexpr int kRowPairs = 8;               // row pairs per batch (16 rows); two batches in flight
constexpr int kMaxHeadsPerPass = 8;

struct DecodeParams {
    const uint16_t *q;        // bf16 [B, H, D]
    const uint16_t *kc;       // bf16 [rows, Hkv, D]
    const uint16_t *vc;       // bf16 [rows, Hkv, D]
    const int64_t *offsets;   // [B + 1]
    const int32_t *seqlens;   // [B]
    const int32_t *qpos;      // [B] or nullptr
    const float *wq;          // [D]
    float *part_o;            // [B * maxC * H, D]
    float *part_ml;           // [B * maxC * H, 2]
    float *out;               // [B, H, D]
    unsigned *err;
    int B, H, Hkv, hpg, maxC, max_len;
    int len_add;              // rows attended beyond seqlens[b]: 1 after an append, else 0
    int pairing;              // kPairAdjacent or kPairHalf
    // Paged cache (pages != nullptr): row r of sequence b is row r % page_size of page
    // pages[b * max_pages + r / page_size]; kc / vc are [num_pages, page_size, Hkv, D].
    const int32_t *pages;
    int page_size, max_pages, num_pages;
    float eps;
    float scale_log2;         // log2(e) / sqrt(D), times the RoPE variant's logit factor
    RopeFreqs rf;
};

// Device-side bounds of sequence b, with len = seqlens[b] + len_add the rows attended:
// 1 <= len <= max_len and len fits its rows.
__device__ __forceinline__ bool decode_seq_ok(const DecodeParams &p, int b, int &len, long long &off) {
    len = p.seqlens[b] + p.len_add;
    if (p.pages != nullptr) {   // paged: the rows of a sequence are its table's pages
        off = 0;
        const long long cap = static_cast<long long>(p.max_pages) * p.page_size;
        return len >= 1 && len <= p.max_len && static_cast<long long>(len) <= cap;
    }
    off = p.offsets[b];
    const long long cap = p.offsets[b + 1] - off;
    return len >= 1 && len <= p.max_len && static_cast<long long>(len) <= cap && off >= 0;
}

template <int HG>
struct HeadsLog2 {
    static constexpr int value = HG == 1 ? 0 : HG == 2 ? 1 : HG == 4 ? 2 : 3;
};

// Sum HG per-lane partial dot products over the 16 lanes of each half-warp with a
// butterfly that halves the vector at each of the first log2(HG) steps.  Returns the
// full sum for head decode_head_of_lane<HG>(lane); all lanes of a half-warp that share
// that head hold the same value.
template <int HG>
__device__ __forceinline__ float decode_reduce_heads(const float (&v)[HG], int lane) {
    constexpr int LG = HeadsLog2<HG>::value;
    float w[HG];
#pragma unroll
    for (int i = 0; i < HG; ++i) w[i] = v[i];
#pragma unroll
    for (int step = 0; step < 4; ++step) {
        const int m = 8 >> step;
        if (step < LG) {
            const bool upper = (lane & m) != 0;
            const int half = HG >> (step + 1);
#pragma unroll
            for (int i = 0; i < HG / 2; ++i) {
                if (i < half) {
                    const float keep = upper ? w[i + half] : w[i];
                    const float send = upper ? w[i] : w[i + half];
                    w[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                }
            }
        } else {
            w[0] += __shfl_xor_sync(0xffffffffu, w[0], m);
        }
    }
    return w[0];
}

template <int HG>
__device__ __forceinline__ int decode_head_of_lane(int lane) {
    constexpr int LG = HeadsLog2<HG>::value;
    int h = 0;
#pragma unroll
    for (int s = 0; s < LG; ++s)
        if (lane & (8 >> s)) h += HG >> (s + 1);
    return h;
}

template <int HG, bool PAGED>
__global__ void __launch_bounds__(128, (HG <= 4 ? 4 : 1)) decode_split_kernel(const __grid_constant__ DecodeParams p) {
    constexpr int LG = HeadsLog2<HG>::value;
    __shared__ __align__(16) float sq[HG][kHeadDim];
    __shared__ __align__(16) float sbuf[4][kWarpKeys * HG];   // scores / probabilities, then partial O
    __shared__ float sml[4][2][HG];

    const int b = blockIdx.x / p.Hkv;
    const int g = blockIdx.x % p.Hkv;
    const int c = blockIdx.y;
    const int jbase = blockIdx.z * HG;
    int len;
    long long off;
    if (!decode_seq_ok(p, b, len, off)) {
        if (c == 0 && g == 0 && blockIdx.z == 0 && threadIdx.x == 0) atomicOr(p.err, kErrInput);
        return;
    }
    const int k0 = c * kChunk;
    if (k0 >= len) return;
    const int k1 = min(len, k0 + kChunk);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    __shared__ int s_bad;   // a warp met a page id out of range
    if (tid == 0) s_bad = 0;
    const int32_t *ptab = PAGED ? p.pages + static_cast<size_t>(b) * p.max_pages : nullptr;
    const int kw0 = k0 + warp * kWarpKeys;
    int kw1 = min(k1, kw0 + kWarpKeys);
    // Page ids of this warp's rows (at most 17 pages of >= 16 rows cover its 256 rows),
    // one per lane, so a batch finds its page with a shuffle rather than a dependent load.
    // A warp whose pages include an id outside [0, num_pages) reads no rows and poisons the
    // chunk's partial sums, so that the merged output of the sequence is NaN.
    const int wpg0 = PAGED ? kw0 / p.page_size : 0;
    int my_page = 0;
    bool warp_bad = false;
    if constexpr (PAGED) {
        if (kw0 < kw1) {
            const int last = (kw1 - 1) / p.page_size;
            const bool mine = wpg0 + lane <= last;
            if (mine) my_page = ptab[wpg0 + lane];
            warp_bad = __any_sync(0xffffffffu, mine && (my_page < 0 || my_page >= p.num_pages));
            if (warp_bad) kw1 = kw0;
        }
    }
    // Paged: the next 16-row batch's page (relative to wpg0) and row inside that page.
    // The batches of a sweep are loaded in order, 16 rows apart, and a batch never crosses
    // a page (page_size is a multiple of 16), so the cursor advances without a division.
    const int off0 = PAGED ? kw0 - wpg0 * p.page_size : 0;
    int cur_pg = 0, cur_off = off0;

    const int sub = lane & 15;    // elements 8*sub .. 8*sub+7 of a row
    const int rsel = lane >> 4;   // which row of the pair
    const int nrow = max(0, kw1 - kw0);
    float *sw = sbuf[warp];
    const size_t row_stride = static_cast<size_t>(p.Hkv) * kHeadDim;
    const uint16_t *kbase = p.kc + (static_cast<size_t>(off) * p.Hkv + g) * kHeadDim + 8 * sub;
    const uint16_t *vbase = p.vc + (static_cast<size_t>(off) * p.Hkv + g) * kHeadDim + 8 * sub;
    const bool writer = (lane & ((16 >> LG) - 1)) == 0;
    const int my_head = decode_head_of_lane<HG>(lane);

    // Loads of the 16-row batch that starts at logical row `base` (rows past kw1 read
    // as zero).  Contiguous caches index rows directly; paged ones take the page id of the
    // cursor from the lane that holds it.
    auto load_batch = [&](const uint16_t *rbase, int base, uint4 (&dst)[kRowPairs]) {
        if constexpr (PAGED) {
            if (base >= kw1) return;
            const int id = __shfl_sync(0xffffffffu, my_page, cur_pg);   // warp-uniform
            const long long pr = static_cast<long long>(id) * p.page_size + cur_off;
            cur_off += 2 * kRowPairs;
            if (cur_off == p.page_size) {
                cur_off = 0;
                ++cur_pg;
            }
#pragma unroll
            for (int u = 0; u < kRowPairs; ++u) {
                const int row = base + 2 * u + rsel;
                dst[u] = row < kw1 ? ldg_stream_v4(rbase + static_cast<size_t>(pr + 2 * u + rsel) * row_stride)
                                   : make_uint4(0u, 0u, 0u, 0u);
            }
        } else {
#pragma unroll
            for (int u = 0; u < kRowPairs; ++u) {
                const int row = base + 2 * u + rsel;
                dst[u] = row < kw1 ? ldg_stream_v4(rbase + static_cast<size_t>(row) * row_stride)
                                   : make_uint4(0u, 0u, 0u, 0u);
            }
        }
    };
    // the first batch of keys is in flight while the query is prepared
    uint4 kn[kRowPairs];
    load_batch(kbase, kw0, kn);

    // ---- q prologue: RMSNorm + RoPE at the query position, scaled into base-2 logits
    {
        const int ps = p.qpos ? p.qpos[b] : p.seqlens[b];
        const float4 w = reinterpret_cast<const float4 *>(p.wq)[lane];
        for (int jj = warp; jj < HG; jj += 4) {
            const int j = jbase + jj;
            float y[4] = {0.f, 0.f, 0.f, 0.f};
            if (j < p.hpg) {
                const int hq = g * p.hpg + j;
                const uint2 raw = *reinterpret_cast<const uint2 *>(p.q + (static_cast<size_t>(b) * p.H + hq) * kHeadDim + 4 * lane);
                const float x0 = bf16lo(raw.x), x1 = bf16hi(raw.x), x2 = bf16lo(raw.y), x3 = bf16hi(raw.y);
                float ss = x0 * x0 + x1 * x1 + x2 * x2 + x3 * x3;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                const float inv = 1.0f / sqrtf(ss * (1.0f / kHeadDim) + p.eps);
                y[0] = w.x * x0 * inv;
                y[1] = w.y * x1 * inv;
                y[2] = w.z * x2 * inv;
                y[3] = w.w * x3 * inv;
            }
            rope_warp4(y, ps, p.rf, p.pairing, lane);   // warp-uniform: j depends on the warp only
            sq[jj][4 * lane + 0] = y[0] * p.scale_log2;
            sq[jj][4 * lane + 1] = y[1] * p.scale_log2;
            sq[jj][4 * lane + 2] = y[2] * p.scale_log2;
            sq[jj][4 * lane + 3] = y[3] * p.scale_log2;
        }
    }
    __syncthreads();
    if (warp_bad && lane == 0) s_bad = 1;

    float2 qr[HG][4];   // pairs of query elements, for packed two-lane FMAs
#pragma unroll
    for (int jj = 0; jj < HG; ++jj)
#pragma unroll
        for (int e = 0; e < 4; ++e) qr[jj][e] = make_float2(sq[jj][8 * sub + 2 * e], sq[jj][8 * sub + 2 * e + 1]);

    // ---- K sweep: base-2 logits of the HG heads for each key of this warp
    for (int base = kw0; base < kw1; base += 2 * kRowPairs) {
        uint4 kv[kRowPairs];
#pragma unroll
        for (int u = 0; u < kRowPairs; ++u) kv[u] = kn[u];
        load_batch(kbase, base + 2 * kRowPairs, kn);
#pragma unroll
        for (int u = 0; u < kRowPairs; ++u) {
            const uint32_t rw[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
            float2 x[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) x[i] = make_float2(bf16lo(rw[i]), bf16hi(rw[i]));
            float part[HG];
#pragma unroll
            for (int jj = 0; jj < HG; ++jj) {
                float2 acc = __fmul2_rn(qr[jj][0], x[0]);
#pragma unroll
                for (int e = 1; e < 4; ++e) acc = __ffma2_rn(qr[jj][e], x[e], acc);
                part[jj] = acc.x + acc.y;
            }
            const float sfull = decode_reduce_heads<HG>(part, lane);
            const int rl = base + 2 * u + rsel - kw0;   // < kWarpKeys by construction
            if (writer) sw[rl * HG + my_head] = sfull;
        }
    }
    uint4 vn[kRowPairs];
    cur_pg = 0;   // the V sweep reads the same rows again
    cur_off = off0;
    load_batch(vbase, kw0, vn);
    __syncwarp();

    // ---- per-warp softmax statistics; lane handles head lane % HG
    const int nent = nrow * HG;
    float mloc = -INFINITY;
    for (int e = lane; e < nent; e += 32) mloc = fmaxf(mloc, sw[e]);
#pragma unroll
    for (int o = 16; o >= HG; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
    float lloc = 0.f;
    for (int e = lane; e < nent; e += 32) {
        const float pe = ex2_approx(sw[e] - mloc);
        sw[e] = pe;
        lloc += pe;
    }
#pragma unroll
    for (int o = 16; o >= HG; o >>= 1) lloc += __shfl_xor_sync(0xffffffffu, lloc, o);
    __syncwarp();

    // ---- V sweep: weighted sum of this warp's value rows
    float2 acc[HG][4];
#pragma unroll
    for (int jj = 0; jj < HG; ++jj)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[jj][e] = make_float2(0.f, 0.f);
    for (int base = kw0; base < kw1; base += 2 * kRowPairs) {
        uint4 vv[kRowPairs];
#pragma unroll
        for (int u = 0; u < kRowPairs; ++u) vv[u] = vn[u];
        load_batch(vbase, base + 2 * kRowPairs, vn);
#pragma unroll
        for (int u = 0; u < kRowPairs; ++u) {
            const int row = base + 2 * u + rsel;
            if (row < kw1) {
                const float *pr = sw + (row - kw0) * HG;
                float pw[HG];
#pragma unroll
                for (int jj = 0; jj < HG; ++jj) pw[jj] = pr[jj];
                const uint32_t rw[4] = {vv[u].x, vv[u].y, vv[u].z, vv[u].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 vv2 = make_float2(bf16lo(rw[i]), bf16hi(rw[i]));
#pragma unroll
                    for (int jj = 0; jj < HG; ++jj) acc[jj][i] = __ffma2_rn(make_float2(pw[jj], pw[jj]), vv2, acc[jj][i]);
                }
            }
        }
    }
#pragma unroll
    for (int jj = 0; jj < HG; ++jj)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc[jj][e].x += __shfl_xor_sync(0xffffffffu, acc[jj][e].x, 16);
            acc[jj][e].y += __shfl_xor_sync(0xffffffffu, acc[jj][e].y, 16);
        }
    __syncwarp();
    if (rsel == 0) {
#pragma unroll
        for (int jj = 0; jj < HG; ++jj) {
            float4 *dst = reinterpret_cast<float4 *>(sw + jj * kHeadDim + 8 * sub);
            dst[0] = make_float4(acc[jj][0].x, acc[jj][0].y, acc[jj][1].x, acc[jj][1].y);
            dst[1] = make_float4(acc[jj][2].x, acc[jj][2].y, acc[jj][3].x, acc[jj][3].y);
        }
    }
    if (lane < HG) {
        sml[warp][0][lane] = mloc;
        sml[warp][1][lane] = lloc;
    }
    __syncthreads();

    // ---- merge the four warps; thread tid owns element d = tid
    const size_t slot0 = (static_cast<size_t>(b) * p.maxC + c) * p.H + static_cast<size_t>(g) * p.hpg;
    if (PAGED && s_bad) {
        if (tid < HG && jbase + tid < p.hpg) {
            p.part_ml[2 * (slot0 + jbase + tid)] = 0.f;
            p.part_ml[2 * (slot0 + jbase + tid) + 1] = __int_as_float(0x7fc00000);
        }
        if (tid == 0) atomicOr(p.err, kErrInput);
        return;
    }
#pragma unroll 1
    for (int jj = 0; jj < HG; ++jj) {
        const int j = jbase + jj;
        if (j >= p.hpg) break;
        float M = sml[0][0][jj];
#pragma unroll
        for (int w = 1; w < 4; ++w) M = fmaxf(M, sml[w][0][jj]);
        float O = 0.f, L = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float sc = ex2_approx(sml[w][0][jj] - M);
            O = fmaf(sc, sbuf[w][jj * kHeadDim + tid], O);
            L = fmaf(sc, sml[w][1][jj], L);
        }
        const size_t slot = slot0 + j;
        p.part_o[slot * kHeadDim + tid] = O;
        if (tid == 0) {
            p.part_ml[2 * slot] = M;
            p.part_ml[2 * slot + 1] = L;
        }
    }
}

__global__ void __launch_bounds__(128) decode_merge_kernel(const __grid_constant__ DecodeParams p) {
    const int b = blockIdx.x / p.H;
    const int hq = blockIdx.x % p.H;
    const int d = threadIdx.x;
    float *o = p.out + (static_cast<size_t>(b) * p.H + hq) * kHeadDim;
    int len;
    long long off;
    if (!decode_seq_ok(p, b, len, off)) {
        o[d] = __int_as_float(0x7fc00000);   // quiet NaN
        return;
    }
    const int nch = (len + kChunk - 1) / kChunk;
    const size_t slot0 = static_cast<size_t>(b) * p.maxC * p.H + hq;   // chunk c: slot0 + c * H
    float M = -INFINITY;
    for (int c = 0; c < nch; ++c) M = fmaxf(M, p.part_ml[2 * (slot0 + static_cast<size_t>(c) * p.H)]);
    float O = 0.f, L = 0.f;
    for (int c = 0; c < nch; ++c) {
        const size_t slot = slot0 + static_cast<size_t>(c) * p.H;
        const float sc = ex2_approx(p.part_ml[2 * slot] - M);
        O = fmaf(sc, p.part_o[slot * kHeadDim + d], O);
        L = fmaf(sc, p.part_ml[2 * slot + 1], L);
    }
    o[d] = O / L;
}

struct AppendParams {
    const uint16_t *k_new;    // bf16 [B, Hkv, D]
    const uint16_t *v_new;    // bf16 [B, Hkv, D]
    uint16_t *kc;             // bf16 [rows, Hkv, D]
    uint16_t *vc;             // bf16 [rows, Hkv, D]
    const int64_t *offsets;   // [B + 1]
    const int32_t *seqlens;   // [B], rows cached before the step
    const int32_t *qpos;      // [B] or nullptr (position = seqlens[b])
    const float *wk;          // [D]
    unsigned *err;
    int B, Hkv, max_len;
    int pairing;              // kPairAdjacent or kPairHalf
    const int32_t *pages;     // paged cache (as DecodeParams), or nullptr
    int page_size, max_pages, num_pages;
    float eps;
    RopeFreqs rf;
};

// One warp per (sequence, KV head): RMSNorm + RoPE of the new key at the token's
// position, rounded to bf16, written to row seqlens[b] of the sequence (in its page, for
// a paged cache); the new value is copied next to it.  Lane l holds elements 4l .. 4l+3.
// A sequence whose rows cannot take the new token is flagged and left untouched.
__global__ void __launch_bounds__(128) decode_append_kernel(const __grid_constant__ AppendParams p) {
    const int lane = threadIdx.x & 31;
    const long long pair = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
    if (pair >= static_cast<long long>(p.B) * p.Hkv) return;
    const int b = static_cast<int>(pair / p.Hkv);
    const int g = static_cast<int>(pair % p.Hkv);
    const int len = p.seqlens[b];
    long long row;   // physical cache row that receives the new token
    if (p.pages != nullptr) {
        const long long cap = static_cast<long long>(p.max_pages) * p.page_size;
        const int id = (len >= 0 && static_cast<long long>(len) < cap) ? p.pages[static_cast<size_t>(b) * p.max_pages +
                                                                                  len / p.page_size]
                                                                       : -1;
        if (!(len >= 0 && len + 1 <= p.max_len && id >= 0 && id < p.num_pages)) {
            if (g == 0 && lane == 0) atomicOr(p.err, kErrInput);
            return;
        }
        row = static_cast<long long>(id) * p.page_size + len % p.page_size;
    } else {
        const long long off = p.offsets[b];
        const long long cap = p.offsets[b + 1] - off;
        if (!(len >= 0 && len + 1 <= p.max_len && static_cast<long long>(len) + 1 <= cap && off >= 0)) {
            if (g == 0 && lane == 0) atomicOr(p.err, kErrInput);
            return;
        }
        row = off + len;
    }
    const int ps = p.qpos ? p.qpos[b] : len;
    const size_t src = (static_cast<size_t>(b) * p.Hkv + g) * kHeadDim + 4 * lane;
    const size_t dst = (static_cast<size_t>(row) * p.Hkv + g) * kHeadDim + 4 * lane;
    const uint2 raw = *reinterpret_cast<const uint2 *>(p.k_new + src);
    const uint2 vraw = *reinterpret_cast<const uint2 *>(p.v_new + src);
    const float x0 = bf16lo(raw.x), x1 = bf16hi(raw.x), x2 = bf16lo(raw.y), x3 = bf16hi(raw.y);
    float ss = x0 * x0 + x1 * x1 + x2 * x2 + x3 * x3;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = 1.0f / sqrtf(ss * (1.0f / kHeadDim) + p.eps);
    const float4 w = reinterpret_cast<const float4 *>(p.wk)[lane];
    float y[4] = {w.x * x0 * inv, w.y * x1 * inv, w.z * x2 * inv, w.w * x3 * inv};
    rope_warp4(y, ps, p.rf, p.pairing, lane);
    uint2 o;
    o.x = pack_bf16x2(y[0], y[1]);
    o.y = pack_bf16x2(y[2], y[3]);
    *reinterpret_cast<uint2 *>(p.kc + dst) = o;
    *reinterpret_cast<uint2 *>(p.vc + dst) = vraw;
}

}  // namespace gqa
