// prefill.cuh -- prefill kernels for sm_100a.
//
//  (1) k_prologue_kernel: RMSNorm + RoPE of every K head vector, written once as
//      bf16 k-hat.  Every K tile is read by all later query blocks of its sequence and
//      by every query head of its group, so transforming it once is cheaper than
//      redoing it in each reader (that would multiply the work by h * (T/128) / 2).
//  (2) attn_fwd_kernel: flash-style causal GQA attention, persistent: one CTA per SM
//      walks work units, a unit being (sequence, KV head, 128-token query block, pair
//      of query heads of the group).  The raw Q tiles are loaded by TMA and normed +
//      rotated in registers in place (the fused q prologue); K-hat/V tiles stream
//      through a TMA ring and serve both query heads of the pair; S = Q K^T and
//      O += P V run on the 5th-generation tensor cores (tcgen05.mma, fp32 accumulators
//      in TMEM); the online softmax runs in two warpgroups (one per head of the pair,
//      ping-ponging with the tensor core) with one query row per thread; causal tiles
//      above the diagonal are never loaded.
//  Both kernels take the RoPE pairing (adjacent or rotate-half) as a template
//  parameter; the frequencies (plain or scaled) arrive precomputed from the host.
//
// Sources, by page title and section: "Qwen3系列1-理论基础&真实结构" D1-2 (stable
// softmax), D1-4 (softmax(QK^T/sqrt(d)+M)V), D1-5 (causal mask), D2-1 (RMSNorm), D2-2
// (QK-Norm then RoPE, V untouched), D2-3 (GQA); "深入剖析Qwen3模型架构" 3.1.2 (K/V
// shared by the h = H/Hkv consecutive query heads, RoPE pairs), 3.4.1 (frequencies);
// "Qwen3" walkthrough, "Attention 的 Forward 流程" (norm, rotary, then attention).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "ptx.cuh"
#include "rope.cuh"

namespace gqa {

// ============================================================================ K prologue
// RoPE cos/sin table: float4 entry (cos, sin, cos, sin) of RoPE pairs 2*i2 and 2*i2+1 of
// flattened token n.  Blocked by 128 tokens, pair-major inside a block, so the 32 threads
// of a warp (consecutive tokens) read 512 contiguous bytes per load in the q prologue.
// Size: round_up(N, 128) * 32 float4.
__host__ __device__ __forceinline__ size_t rope_table_index(long long n, int i2) {
    return (static_cast<size_t>(n >> 7) * 32 + static_cast<size_t>(i2)) * 128 + static_cast<size_t>(n & 127);
}

struct KPrologueParams {
    const uint16_t *k;     // bf16: the Hkv head vectors of token n start at k + n * k_stride
    const uint16_t *v;     // bf16 values copied beside k-hat (v + n * v_stride), or nullptr
    const int32_t *pos;    // [ntok]
    const float *wk;       // [D]
    uint16_t *khat;        // bf16 [rows, Hkv, D]: token n goes to row dst_row(n)
    uint16_t *vout;        // bf16 [rows, Hkv, D] (with v), or nullptr
    float *rope_cs;        // RoPE cos/sin of every token in the blocked table layout (rope_table_index), or nullptr
    // Destination rows.  cu == nullptr: token n -> row n.  Otherwise token n of sequence b
    // (cu[b] <= n < cu[b+1]) -> row cache_off[b] + prefix[b] + n - cu[b], which must lie
    // inside the sequence's rows cache_off[b] .. cache_off[b+1] - 1 (else the token is not
    // written and the device status records an input error).
    const int64_t *cu;        // [B + 1]
    const int64_t *cache_off; // [B + 1]
    const int32_t *prefix;    // [B]
    // Paged destination (pages != nullptr, with cu): the token's row in its sequence,
    // prefix[b] + n - cu[b], is row r % page_size of page pages[b * max_pages + r / page_size].
    const int32_t *pages;
    int page_size, max_pages, num_pages;
    unsigned *err;
    long long ntok, k_stride, v_stride, rows;
    int Hkv, B;
    float eps;
    RopeFreqs rf;
};

// Destination row of token n, or -1 if the sequence geometry puts it out of range.
__device__ __forceinline__ long long k_prologue_row(const KPrologueParams &p, long long n) {
    if (p.cu == nullptr) return n;
    int lo = 0, hi = p.B;   // largest b with cu[b] <= n
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.cu[mid] <= n) lo = mid;
        else hi = mid;
    }
    const long long c0 = p.cu[lo], c1 = p.cu[lo + 1];
    const long long pre = p.prefix[lo];
    if (p.pages != nullptr) {
        const long long r = pre + (n - c0), pg = r / p.page_size;
        if (!(c0 <= n && n < c1 && pre >= 0 && pg < p.max_pages)) return -1;
        const int id = p.pages[static_cast<long long>(lo) * p.max_pages + pg];
        if (id < 0 || id >= p.num_pages) return -1;
        return static_cast<long long>(id) * p.page_size + (r - pg * p.page_size);
    }
    const long long r0 = p.cache_off[lo], r1 = p.cache_off[lo + 1];
    const long long row = r0 + pre + (n - c0);
    if (!(c0 <= n && n < c1 && pre >= 0 && r0 >= 0 && row < r1 && r1 <= p.rows)) return -1;
    return row;
}

// One warp per token at a time; each half-warp transforms one head vector, each lane
// eight consecutive elements.  Adjacent pairing: the lane's elements are four RoPE pairs.
// Rotate-half pairing: lane j < 8 holds elements 8j .. 8j+7, whose partners 64 + 8j ..
// sit in lane j + 8; both rotate by the frequencies 8j .. 8j+7.  Each lane evaluates the
// cos/sin of four frequencies once per token (reused for all of the token's KV heads,
// exchanged with the partner lane for rotate-half) and optionally stores them so the
// query side (same positions) can read them instead of evaluating them again.
template <int PAIRING>
__global__ void __launch_bounds__(256) k_prologue_kernel(const __grid_constant__ KPrologueParams p) {
    const int lane = threadIdx.x & 31;
    const int half = lane >> 4;
    const int sub = lane & 15;
    const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    long long tok = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;

    const float4 wa = reinterpret_cast<const float4 *>(p.wk)[2 * sub];
    const float4 wb = reinterpret_cast<const float4 *>(p.wk)[2 * sub + 1];
    const float w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};

    constexpr bool half_pairs = PAIRING == kPairHalf;
    // frequencies this lane evaluates: 4 sub .. 4 sub + 3 (adjacent), or 8 (sub & 7) +
    // 4 (sub >> 3) + 0..3 (rotate-half: the partner lane evaluates the other four)
    const int f0 = half_pairs ? 8 * (sub & 7) + 4 * (sub >> 3) : 4 * sub;

    for (; tok < p.ntok; tok += nwarps) {
        const long long drow = k_prologue_row(p, tok);
        if (drow < 0) {
            if (lane == 0) atomicOr(p.err, kErrInput);
            continue;
        }
        const int ps = p.pos[tok];
        float cs[8], sn[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) rope_cos_sin(ps, p.rf.inv_freq[f0 + i], cs[i], sn[i]);
        if (p.rope_cs != nullptr && half == 0) {
            float4 *tab = reinterpret_cast<float4 *>(p.rope_cs);
            tab[rope_table_index(tok, f0 / 2)] = make_float4(cs[0], sn[0], cs[1], sn[1]);
            tab[rope_table_index(tok, f0 / 2 + 1)] = make_float4(cs[2], sn[2], cs[3], sn[3]);
        }
        if constexpr (half_pairs) {   // cos/sin of frequencies 8 (sub & 7) + 0..7, in that order
            float pc[4], ps4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                pc[i] = __shfl_xor_sync(0xffffffffu, cs[i], 8);
                ps4[i] = __shfl_xor_sync(0xffffffffu, sn[i], 8);
            }
            if (sub >= 8) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    cs[4 + i] = cs[i];
                    sn[4 + i] = sn[i];
                    cs[i] = pc[i];
                    sn[i] = ps4[i];
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    cs[4 + i] = pc[i];
                    sn[4 + i] = ps4[i];
                }
            }
        }
        // up to 8 head pairs per batch: all loads first, so they are in flight together
        for (int h0 = 0; h0 < p.Hkv; h0 += 16) {
            constexpr int kPairs = 8;
            uint4 raw[kPairs];
#pragma unroll
            for (int u = 0; u < kPairs; ++u) {
                const int hh = h0 + 2 * u + half;
                raw[u] = make_uint4(0u, 0u, 0u, 0u);
                if (hh < p.Hkv)
                    raw[u] = *reinterpret_cast<const uint4 *>(p.k + static_cast<size_t>(tok) * p.k_stride +
                                                              static_cast<size_t>(hh) * kHeadDim + 8 * sub);
            }
#pragma unroll
            for (int u = 0; u < kPairs; ++u) {
                const int hh = h0 + 2 * u + half;
                if (h0 + 2 * u >= p.Hkv) break;   // warp-uniform
                const uint32_t rw[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
                float x[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    x[2 * i] = bf16lo(rw[i]);
                    x[2 * i + 1] = bf16hi(rw[i]);
                }
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
                for (int o = 8; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                const float inv = 1.0f / sqrtf(ss * (1.0f / kHeadDim) + p.eps);
                uint32_t outw[4];
                if constexpr (!half_pairs) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float a = w[2 * i] * x[2 * i] * inv;
                        const float b = w[2 * i + 1] * x[2 * i + 1] * inv;
                        outw[i] = pack_bf16x2(a * cs[i] - b * sn[i], a * sn[i] + b * cs[i]);
                    }
                } else {
                    const float sign = sub < 8 ? -1.0f : 1.0f;   // first half: a c - b s; second: a c + b s
                    float y[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float a = w[e] * x[e] * inv;
                        const float b = __shfl_xor_sync(0xffffffffu, a, 8);
                        y[e] = fmaf(sign * b, sn[e], a * cs[e]);
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i) outw[i] = pack_bf16x2(y[2 * i], y[2 * i + 1]);
                }
                if (hh < p.Hkv)
                    *reinterpret_cast<uint4 *>(p.khat + (static_cast<size_t>(drow) * p.Hkv + hh) * kHeadDim + 8 * sub) =
                        make_uint4(outw[0], outw[1], outw[2], outw[3]);
            }
        }
        if (p.v != nullptr) {   // the token's values go beside its keys
            for (int hh = half; hh < p.Hkv; hh += 2)
                *reinterpret_cast<uint4 *>(p.vout + (static_cast<size_t>(drow) * p.Hkv + hh) * kHeadDim + 8 * sub) =
                    *reinterpret_cast<const uint4 *>(p.v + static_cast<size_t>(tok) * p.v_stride +
                                                     static_cast<size_t>(hh) * kHeadDim + 8 * sub);
        }
    }
}

// ============================================================================ attention
constexpr int kBM = 128;                       // query rows per tile (one per softmax thread)
constexpr int kBN = 128;                       // keys per K/V tile
constexpr int kStages = 4;                     // K/V ring depth (tiles)
constexpr uint32_t kTileBytes = 128 * 128 * 2; // one bf16 128x128 tile
constexpr uint32_t kBoxBytes = 128 * 128;      // 128 rows x 64 bf16 (one 128-byte swizzle span)
constexpr uint32_t kStageBytes = 128 * 32 * 4; // epilogue staging per head: 128 rows x 32 fp32 columns
constexpr uint32_t kOffQ = 0;                                   // 2 tiles
constexpr uint32_t kOffKV = kOffQ + 2 * kTileBytes;             // kStages tiles
constexpr uint32_t kOffStage = kOffKV + kStages * kTileBytes;   // 2 staging buffers
constexpr uint32_t kOffBar = kOffStage + 2 * kStageBytes;
enum {
    BAR_Q_FULL = 0,    // [2] TMA -> softmax WG: raw Q tile landed
    BAR_Q_READY = 2,   // [2] softmax WG -> MMA: Q tile normed + rotated in place (128 arrivals)
    BAR_Q_EMPTY = 4,   // [2] MMA (commit) -> TMA: the unit's last Q K^T on the slot finished
    BAR_K0_FULL = 6,   // TMA -> MMA: the first K tile of a unit landed
    BAR_KV_EMPTY = 7,                // [kStages] MMA (commit) -> TMA
    BAR_S_FULL = 7 + kStages,        // [2] MMA (commit) -> softmax WG: S of the next tile is in TMEM
    BAR_P_FULL = 9 + kStages,        // [2] softmax WG -> MMA: P written over S in TMEM, O rescaled (128 arrivals)
    BAR_O_FULL = 11 + kStages,       // [2] MMA (commit) -> softmax WG: the unit's last P V finished
    BAR_O_EMPTY = 13 + kStages,      // [2] softmax WG -> MMA: O read out by the epilogue (128 arrivals)
    BAR_DRAIN = 15 + kStages,        // MMA drains its own work before TMEM is released
    BAR_STEP_FULL = 16 + kStages,    // [3] TMA -> MMA: V_j and K_{j+1} landed (one wait per tile)
    BAR_NEVER = 19 + kStages,        // never signalled: the failure-path test waits on it
    NUM_BARS = 20 + kStages
};
constexpr uint32_t kOffTmemSlot = kOffBar + NUM_BARS * 8;
constexpr uint32_t kSmemBytes = kOffTmemSlot + 16 + 1024;  // + slack to align the base to 1024
// TMEM: S0 | S1 | O0 | O1, 128 fp32 columns each.  P of a tile (bf16, two per column)
// is written over the first 64 columns of its S once S has been read.
constexpr uint32_t kTmemCols = 512;
constexpr int kAttnThreads = 384;     // warp 0 TMA, warp 1 MMA, warps 4-7 / 8-11 softmax
static_assert(kSmemBytes <= 232448, "shared memory budget");
// Registers per thread: launched at kRegsLaunch (384 threads x 168 = 64512 of the SM's
// 65536), then warpgroup 0 (TMA, MMA and two idle warps) gives up registers to the two
// softmax warpgroups, whose 128-column score rows need them.
constexpr uint32_t kRegsLaunch = 168, kRegsCtl = 120, kRegsSoftmax = 192;
static_assert(kRegsCtl * 128 + 2 * kRegsSoftmax * 128 <= kRegsLaunch * kAttnThreads, "register split");

// Geometry of a prefill launch.  Sequence b has len(b) query tokens, rows q0(b) ..
// q0(b) + len(b) - 1 of q / pos / out, and prefix(b) + len(b) keys, rows kv0(b) .. of
// k-hat / v, the first prefix(b) of them cached before these queries.  Query row t of
// the sequence is token prefix(b) + t and sees keys 0 .. prefix(b) + t (causal on the
// token index).  Dense prefill: q0 = kv0 = b T, len = T, prefix = 0 (no arrays).
struct AttnParams {
    const int32_t *pos;    // [Nq]
    const float *rope_cs;  // RoPE cos/sin table over the Nq query tokens (rope_table_index), or nullptr (evaluate here)
    const float *wq;       // [D]
    void *out;             // [Nq, H, D], fp32 or (out_bf16) bf16
    unsigned *err;
    const int64_t *cu_q;   // [B + 1] query-row offsets, or nullptr: b T
    const int64_t *kv_off; // [B] first K/V row, or nullptr: the query-row offset
    const int32_t *prefix; // [B] cached keys before the first query token, or nullptr: 0
    // Paged K/V (kv_pages != nullptr): key row r of sequence b is row r % kv_page_size of page
    // kv_pages[b * kv_max_pages + r / kv_page_size]; the tensor maps cover the pages' rows,
    // in boxes of min(kv_page_size, 128) rows.
    const int32_t *kv_pages;
    int kv_page_size, kv_max_pages, kv_num_pages;
    int kv_segs;           // page segments of a tile: 128 / kv_page_size, or 1 when a page holds whole tiles
    int kv_seg_rows;       // rows of a segment: 128 / kv_segs
    long long nq_rows;     // rows of q / pos / out
    long long nkv_rows;    // rows of k-hat / v (paged: rows a sequence can address, kv_max_pages * kv_page_size)
    int B, T, H, Hkv, hpg, nqb, npairs, nunits;
    int band;              // KV groups (sequence, KV head) scheduled together: their K/V fit in L2
    // Packed inputs: the (sequence, query block) pairs that have work, in schedule order
    // (unit_list_kernel), each standing for uexp = Hkv * npairs units, and their count.
    const int2 *ulist;     // or nullptr: every unit of the band order has work
    const int *ulist_n;
    int uexp;
    int out_bf16;          // 1: the output is rounded to bf16 (the input of the output projection)
    int test_stall;        // 1 (failure-path test only): the MMA thread first waits on BAR_NEVER
    float eps;
    float scale_log2;      // log2(e) / sqrt(D) times the RoPE variant's logit factor: softmax runs in base 2
    RopeFreqs rf;
};

// One work unit: a 128-row query block of one sequence and a pair of query heads of a
// KV group.  Units are numbered band by band, where a band is `band` consecutive KV groups
// (sequence, KV head) whose K/V together fit in L2, and inside a band heaviest (latest query
// block) first: the CTAs running at the same time then read the same K/V tiles, which stay
// in L2, instead of streaming every group's K/V through it.
struct AttnUnit {
    long long q0;     // query row of block row 0 (q0(b) + qb * 128)
    long long kv0;    // K/V row of key 0
    int b, g, hq0, nslots;
    int rows;         // valid rows of the block (<= 128)
    int key0;         // token index of block row 0 (prefix + qb * 128)
    int n_kv;         // K/V tiles the block reads: keys 0 .. key0 + rows - 1
};

// Decode unit u; false when it has no work (a query block past the end of a shorter
// sequence, or a sequence whose device-side geometry is out of range).
// Unit u of a listed launch: (sequence, query block, KV head, head pair).  Kept out of line:
// its divisions would otherwise hold registers in every role that decodes units.
__device__ __noinline__ int4 listed_unit(const int2 *list, int uexp, int npairs, int u) {
    const int e = u / uexp, r = u - e * uexp;
    const int2 ent = list[e];
    const int g = r / npairs;
    return make_int4(ent.x, ent.y, g, r - g * npairs);
}

template <bool LISTED>
__device__ __forceinline__ bool attn_unit(const AttnParams &p, int u, AttnUnit &w, bool &bad) {
    bad = false;
    int qb, pair;
    if constexpr (LISTED) {
        // u -> (listed sequence and query block, KV head, head pair)
        const int4 d = listed_unit(p.ulist, p.uexp, p.npairs, u);
        w.b = d.x;
        qb = d.y;
        w.g = d.z;
        pair = d.w;
    } else {
        // u -> (band of KV groups, query block latest first, group in the band, head pair)
        const int ngroups = p.B * p.Hkv;
        const int per_band = p.band * p.nqb * p.npairs;
        const int band = u / per_band;
        const int gb = min(p.band, ngroups - band * p.band);   // groups in this band
        int rem = u - band * per_band;
        qb = p.nqb - 1 - rem / (gb * p.npairs);
        rem %= gb * p.npairs;
        pair = rem % p.npairs;
        const int gi = band * p.band + rem / p.npairs;
        w.g = gi % p.Hkv;
        w.b = gi / p.Hkv;
    }
    long long q0 = static_cast<long long>(w.b) * p.T, len = p.T;
    if (p.cu_q != nullptr) {
        q0 = p.cu_q[w.b];
        len = p.cu_q[w.b + 1] - q0;
    }
    const long long kv0 = p.kv_pages != nullptr ? 0 : p.kv_off != nullptr ? p.kv_off[w.b] : q0;
    const long long pre = p.prefix != nullptr ? p.prefix[w.b] : 0;
    if (q0 < 0 || len < 0 || q0 + len > p.nq_rows || len > static_cast<long long>(p.nqb) * kBM || pre < 0 ||
        kv0 < 0 || kv0 + pre + len > p.nkv_rows || pre + len > 0x7fff0000LL) {
        bad = true;
        return false;
    }
    if (static_cast<long long>(qb) * kBM >= len) return false;
    w.q0 = q0 + static_cast<long long>(qb) * kBM;
    w.kv0 = kv0;
    w.rows = static_cast<int>(min(static_cast<long long>(kBM), len - static_cast<long long>(qb) * kBM));
    w.key0 = static_cast<int>(pre) + qb * kBM;
    w.n_kv = (w.key0 + w.rows - 1) / kBN + 1;
    w.nslots = min(2, p.hpg - 2 * pair);
    w.hq0 = w.g * p.hpg + 2 * pair;
    return true;
}

// Shared-memory address of 16-byte chunk c (0..15, i.e. elements 8c..8c+7) of row r of
// a 128x128 bf16 tile stored as two 128B-swizzled boxes of 64 columns.
__device__ __forceinline__ uint32_t tile_chunk_addr(uint32_t tile, int r, int c) {
    return tile + static_cast<uint32_t>(c >> 3) * kBoxBytes + static_cast<uint32_t>(r) * 128u +
           (static_cast<uint32_t>((c & 7) ^ (r & 7)) << 4);
}

// S = Q K^T for one 128x128 tile: eight K=16 steps over the head dimension, both
// operands K-major in shared memory.
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t sq, uint32_t sk, uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = static_cast<uint32_t>(kk >> 2) * kBoxBytes + static_cast<uint32_t>(kk & 3) * 32u;
        umma_bf16_ss(d_tmem, sw128_desc(sq + off, 16, 1024), sw128_desc(sk + off, 16, 1024), idesc,
                     kk > 0 ? 1u : 0u);
    }
}

// O (+)= P V: eight K=16 steps over the keys.  P (bf16, K-major) is read from tensor
// memory, 8 columns per step; V is MN-major in shared memory (head dim contiguous):
// its two 64-column boxes are kBoxBytes apart (LBO) and 8-key groups 1024 bytes (SBO).
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t sv, uint32_t idesc,
                                         bool accumulate) {
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint32_t offv = static_cast<uint32_t>(kk) * 2048u;
        umma_bf16_ts(d_tmem, p_tmem + 8u * kk, sw128_desc(sv + offv, kBoxBytes, 1024), idesc,
                     (accumulate || kk > 0) ? 1u : 0u);
    }
}

// RMSNorm (w_q, eps) and RoPE of query row r (flattened token n) of a raw Q tile, in
// place, with adjacent or rotate-half pairing.  The rotation uses the K prologue's
// cos/sin table when given (coalesced across the warp: consecutive rows are consecutive
// tokens), fetched in batches of 16 (adjacent) or 8 (rotate-half) loads, else evaluates
// cos/sin from the position ps.
template <int PAIRING>
__device__ __forceinline__ void transform_q_row(uint32_t sq, int r, int ps, const float *table, long long n,
                                                const float *wq, float eps, const RopeFreqs &rf) {
    float sq8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // eight short chains, not one of 128
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const uint4 v = ld_shared_v4(tile_chunk_addr(sq, r, c));
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float a = bf16lo(u[i]), b = bf16hi(u[i]);
            sq8[2 * i] = fmaf(a, a, sq8[2 * i]);
            sq8[2 * i + 1] = fmaf(b, b, sq8[2 * i + 1]);
        }
    }
    const float ss = ((sq8[0] + sq8[1]) + (sq8[2] + sq8[3])) + ((sq8[4] + sq8[5]) + (sq8[6] + sq8[7]));
    const float inv = 1.0f / sqrtf(ss * (1.0f / kHeadDim) + eps);
    if constexpr (PAIRING == kPairHalf) {
        // rotate-half: chunk c (elements 8c .. 8c+7, c < 8) meets chunk c + 8, at the
        // frequencies 8c .. 8c+7; four batches of 16 frequencies (8 table entries)
#pragma unroll 1
        for (int qt = 0; qt < 4; ++qt) {
            float4 tb[8];   // (cos, sin) of frequencies 16 qt .. 16 qt + 15, two per float4
            if (table != nullptr) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    tb[i] = __ldg(reinterpret_cast<const float4 *>(table) + rope_table_index(n, 8 * qt + i));
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int f = 16 * qt + 2 * i;
                    rope_cos_sin(ps, rf.inv_freq[f], tb[i].x, tb[i].y);
                    rope_cos_sin(ps, rf.inv_freq[f + 1], tb[i].z, tb[i].w);
                }
            }
#pragma unroll
            for (int c8 = 0; c8 < 2; ++c8) {
                const int c = 2 * qt + c8;
                const uint32_t addr1 = tile_chunk_addr(sq, r, c), addr2 = tile_chunk_addr(sq, r, c + 8);
                const uint4 v1 = ld_shared_v4(addr1), v2 = ld_shared_v4(addr2);
                const uint32_t u1[4] = {v1.x, v1.y, v1.z, v1.w}, u2[4] = {v2.x, v2.y, v2.z, v2.w};
                const float4 w1a = __ldg(reinterpret_cast<const float4 *>(wq) + 2 * c);
                const float4 w1b = __ldg(reinterpret_cast<const float4 *>(wq) + 2 * c + 1);
                const float4 w2a = __ldg(reinterpret_cast<const float4 *>(wq) + 2 * c + 16);
                const float4 w2b = __ldg(reinterpret_cast<const float4 *>(wq) + 2 * c + 17);
                const float w1[8] = {w1a.x, w1a.y, w1a.z, w1a.w, w1b.x, w1b.y, w1b.z, w1b.w};
                const float w2[8] = {w2a.x, w2a.y, w2a.z, w2a.w, w2b.x, w2b.y, w2b.z, w2b.w};
                uint32_t o1[4], o2[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 t = tb[4 * c8 + i];   // frequencies 8c + 2i, 8c + 2i + 1
                    const float a0 = w1[2 * i] * bf16lo(u1[i]) * inv, a1 = w1[2 * i + 1] * bf16hi(u1[i]) * inv;
                    const float b0 = w2[2 * i] * bf16lo(u2[i]) * inv, b1 = w2[2 * i + 1] * bf16hi(u2[i]) * inv;
                    o1[i] = pack_bf16x2(a0 * t.x - b0 * t.y, a1 * t.z - b1 * t.w);
                    o2[i] = pack_bf16x2(b0 * t.x + a0 * t.y, b1 * t.z + a1 * t.w);
                }
                st_shared_v4(addr1, make_uint4(o1[0], o1[1], o1[2], o1[3]));
                st_shared_v4(addr2, make_uint4(o2[0], o2[1], o2[2], o2[3]));
            }
        }
    } else {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        float4 tb[16];   // (cos, sin) of pairs 32*half .. 32*half+31, two pairs per float4
        if (table != nullptr) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                tb[i] = __ldg(reinterpret_cast<const float4 *>(table) + rope_table_index(n, 16 * half + i));
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int pr = 32 * half + 2 * i;
                rope_cos_sin(ps, rf.inv_freq[pr], tb[i].x, tb[i].y);
                rope_cos_sin(ps, rf.inv_freq[pr + 1], tb[i].z, tb[i].w);
            }
        }
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
            const int c = 8 * half + c8;   // elements 8c..8c+7 = RoPE pairs 4c..4c+3
            const uint32_t addr = tile_chunk_addr(sq, r, c);
            const uint4 v = ld_shared_v4(addr);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
            const float4 wa = __ldg(reinterpret_cast<const float4 *>(wq) + 2 * c);
            const float4 wb = __ldg(reinterpret_cast<const float4 *>(wq) + 2 * c + 1);
            const float w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
            const float cs[4] = {tb[2 * c8].x, tb[2 * c8].z, tb[2 * c8 + 1].x, tb[2 * c8 + 1].z};
            const float sn[4] = {tb[2 * c8].y, tb[2 * c8].w, tb[2 * c8 + 1].y, tb[2 * c8 + 1].w};
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float a = w[2 * i] * bf16lo(u[i]) * inv;
                const float b = w[2 * i + 1] * bf16hi(u[i]) * inv;
                o[i] = pack_bf16x2(a * cs[i] - b * sn[i], a * sn[i] + b * cs[i]);
            }
            st_shared_v4(addr, make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
    }
}

// 2^(x*scale + negm) of 64 consecutive scores, packed as bf16 pairs into 32 words; their
// (unrounded) sum goes into eight partial sums.
__device__ __forceinline__ void exp_pack64(const float *x, float scale, float negm, uint32_t *pk, float (&sp)[8]) {
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        const float e0 = ex2_approx(fmaf(x[2 * c], scale, negm));
        const float e1 = ex2_approx(fmaf(x[2 * c + 1], scale, negm));
        sp[(2 * c) & 7] += e0;
        sp[(2 * c + 1) & 7] += e1;
        pk[c] = pack_bf16x2(e0, e1);
    }
}

// P of a 128-key tile into TMEM (over S): keys 0-63, then 64-127.
__device__ __forceinline__ void exp_tile(const float *x, float scale, float negm, uint32_t tS, float (&sp)[8]) {
    {
        uint32_t pk[32];
        exp_pack64(x, scale, negm, pk, sp);
        tmem_st32(tS, reinterpret_cast<const float *>(pk));
    }
    {
        uint32_t pk[32];
        exp_pack64(x + 64, scale, negm, pk, sp);
        tmem_st32(tS + 32, reinterpret_cast<const float *>(pk));
    }
}

__device__ __forceinline__ float max8(const float (&m)[8]) {
    return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])), fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
}

// Units of the launch: those listed for packed inputs (the count comes from the list kernel
// that ran before on the stream), else every unit of the band order.
template <bool LISTED>
__device__ __forceinline__ int attn_unit_count(const AttnParams &p) {
    if constexpr (LISTED) return *p.ulist_n * p.uexp;
    return p.nunits;
}

// Paged K/V: the page id of segment i of 128-key tile j of sequence b.  A tile is kv_segs
// whole pages (up to kMaxSegs, for 16-row pages) or lies inside one page.  A segment past
// the tile, past the last visible key, lim, or past the table's row is not looked up (-1).
// off is the tile's first row inside the page (0 for whole pages).
constexpr int kMaxSegs = 128 / 16;
static_assert(kMaxSegs * 16 == kBN && 2 * kMaxSegs <= 32, "one lane per box of a 16-row-page tile");
__device__ __forceinline__ int kv_page_id(const AttnParams &p, int b, int j, int lim, int i, int &off) {
    const int32_t *row = p.kv_pages + static_cast<long long>(b) * p.kv_max_pages;
    const int key = j * kBN;
    if (p.kv_segs == 1) {
        const int pg = key / p.kv_page_size;
        off = key - pg * p.kv_page_size;
        return (i == 0 && key < lim && pg < p.kv_max_pages) ? __ldg(row + pg) : -1;
    }
    const int pg = j * p.kv_segs + i;
    off = 0;
    return (i < p.kv_segs && pg * p.kv_page_size < lim && pg < p.kv_max_pages) ? __ldg(row + pg) : -1;
}

// The (sequence, query block) pairs of a packed launch that have work, in the order the
// attention kernel deals them out: bands of `band` sequences (whose K/V fit in L2 together),
// inside a band query blocks latest first, then the sequences of the band.  Units past the end
// of a shorter sequence would otherwise leave holes in the rounds of the static schedule.
// One CTA of 1024 threads: each counts the slots of a contiguous range, a block-wide scan
// gives each range its place, and each writes its entries.  A sequence whose bounds are out
// of range gets no entries and sets kErrInput.
__global__ void __launch_bounds__(1024) unit_list_kernel(const int64_t *cu, const int64_t *kv_off, const int32_t *prefix,
                                                       bool kv_paged, long long nq_rows, long long nkv_rows, int B,
                                                       int nqb, int band, int2 *list, int cap, int *count,
                                                       unsigned *err) {
    __shared__ int warp_sum[32];
    const long long per_band = static_cast<long long>(band) * nqb;
    const long long slots = (static_cast<long long>(B) + band - 1) / band * per_band;
    const long long per = (slots + blockDim.x - 1) / blockDim.x;
    const long long s0 = min(slots, per * threadIdx.x), s1 = min(slots, s0 + per);
    // slot s -> (b, qb), or -1 when the slot has no work
    auto slot_block = [&](long long s, int &b) -> int {
        const long long bi = s / per_band, rem = s - bi * per_band;
        const int qb = nqb - 1 - static_cast<int>(rem / band);
        b = static_cast<int>(bi * band + rem % band);
        if (b >= B) return -1;
        const long long q0 = cu[b], len = cu[b + 1] - q0;
        const long long kv0 = kv_paged ? 0 : kv_off != nullptr ? kv_off[b] : q0;
        const long long pre = prefix != nullptr ? prefix[b] : 0;
        if (q0 < 0 || len < 0 || q0 + len > nq_rows || len > static_cast<long long>(nqb) * 128 || pre < 0 ||
            kv0 < 0 || kv0 + pre + len > nkv_rows || pre + len > 0x7fff0000LL) {
            if (qb == 0) atomicOr(err, kErrInput);
            return -1;
        }
        return static_cast<long long>(qb) * 128 < len ? qb : -1;
    };
    int n = 0;
    for (long long s = s0; s < s1; ++s) {
        int b;
        if (slot_block(s, b) >= 0) ++n;
    }
    // exclusive scan of n over the block: within each warp, then over the warp totals
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int incl = n;
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_sum[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int t = lane < static_cast<int>(blockDim.x >> 5) ? warp_sum[lane] : 0;
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += u;
        }
        warp_sum[lane] = t;   // inclusive over warps
    }
    __syncthreads();
    int pos = (wid > 0 ? warp_sum[wid - 1] : 0) + incl - n;
    for (long long s = s0; s < s1; ++s) {
        int b;
        const int qb = slot_block(s, b);
        if (qb < 0) continue;
        // sequences that overlap (cu not ascending) can list more than the buffer holds
        if (pos < cap)
            list[pos] = make_int2(b, qb);
        else
            atomicOr(err, kErrInput);
        ++pos;
    }
    if (threadIdx.x == blockDim.x - 1) *count = min(pos, cap);
}

// The work unit of round r for this CTA.  Units are numbered heaviest first; the rounds
// alternate their direction over the CTAs (snake order), so that each pair of rounds
// gives every CTA about the same causal length.
__device__ __forceinline__ int attn_unit_of_round(int r) {
    const int G = gridDim.x, c = blockIdx.x;
    return r * G + ((r & 1) ? G - 1 - c : c);
}

// Persistent flash-style causal GQA attention: one CTA per SM walks one work unit per
// round (attn_unit_of_round).  The K/V ring, the barrier
// phases and the TMEM buffers carry over from unit to unit, so that the next unit's Q
// and first K/V tiles load, and its Q tile is normed and rotated, while the current
// unit's last P V and epilogue run.  LISTED: the units are those of the unit list
// (packed inputs), else every unit of the band order.
template <int PAIRING, bool LISTED>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw_base & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    const uint32_t sbase = raw_base + pad;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    const uint32_t sQ0 = sbase + kOffQ, sKV0 = sbase + kOffKV;
    const uint32_t bar0 = sbase + kOffBar;
#define BAR(i) (bar0 + 8u * static_cast<uint32_t>(i))

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(BAR(BAR_Q_FULL + s), 1);
            mbar_init(BAR(BAR_Q_READY + s), kBM);
            mbar_init(BAR(BAR_Q_EMPTY + s), 1);
            mbar_init(BAR(BAR_S_FULL + s), 1);
            mbar_init(BAR(BAR_P_FULL + s), kBM);
            mbar_init(BAR(BAR_O_FULL + s), 1);
            mbar_init(BAR(BAR_O_EMPTY + s), kBM);
        }
        mbar_init(BAR(BAR_K0_FULL), 1);
        for (int i = 0; i < kStages; ++i) mbar_init(BAR(BAR_KV_EMPTY + i), 1);
        for (int i = 0; i < 3; ++i) mbar_init(BAR(BAR_STEP_FULL + i), 1);
        mbar_init(BAR(BAR_DRAIN), 1);
        mbar_init(BAR(BAR_NEVER), 1);
        fence_mbarrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(sbase + kOffTmemSlot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + kOffTmemSlot);
    const int nun = attn_unit_count<LISTED>(p);
    if (warp < 4) {
    regs_dec<kRegsCtl>();
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // Lane 0 walks the schedule, waits for free buffers and arms the barriers.  With
        // paged K/V the whole warp walks it: each lane issues one box of a tile (a half of
        // one page segment), so a tile of 16-row pages is one warp instruction, not 16
        // issued one after the other; every lane waits for the buffer it writes itself.
        const bool paged = p.kv_pages != nullptr;
        const unsigned wmask = paged ? 0xffffffffu : 1u;
        if (lane == 0 || paged) {
            bool ok = true;
            uint32_t q_uses[2] = {0u, 0u};   // Q loads per slot so far
            uint32_t k0_uses = 0;            // units so far (first K tiles)
            uint32_t it = 0;                 // K/V ring items so far (K0 V0 K1 V1 ... per unit)
            uint32_t gs = 0;                 // steps so far (one per K/V tile pair)
            uint32_t armed = 0;                     // steps armed so far (step k on barrier k % 3)
            // paged: this lane's box is half (lane & 1) of segment lane >> 1 of the tile
            const int seg_i = lane >> 1, half = lane & 1;
            for (int r = 0; ok; ++r) {
                const int u = attn_unit_of_round(r);
                if (u >= nun) break;
                AttnUnit w;
                bool bad;
                if (!attn_unit<LISTED>(p, u, w, bad)) {
                    if (bad && lane == 0) atomicOr(p.err, kErrInput);
                    continue;
                }
                // paged K/V: the page id of this lane's segment, loaded one tile ahead and
                // used for both K and V; a segment with no visible key is not looked up
                const int kv_lim = w.key0 + w.rows;
                int pid_cur = -1, pid_nxt = -1, poff_cur = 0, poff_nxt = 0;
                if (paged) pid_cur = kv_page_id(p, w.b, 0, kv_lim, seg_i, poff_cur);
                if (lane == 0) {
                    if (p.rope_cs != nullptr) {   // the table blocks holding this query block's tokens
                        for (long long blk = w.q0 >> 7; blk <= ((w.q0 + w.rows - 1) >> 7); ++blk)
                            prefetch_l2_bulk(p.rope_cs + rope_table_index(blk << 7, 0) * 4, 32 * 128 * 16);
                    }
#pragma unroll
                    for (int s = 0; s < 2; ++s) {   // unrolled: the per-slot counters stay in registers
                        if (s >= w.nslots || !ok) break;
                        // the slot is free once the previous unit's last Q K^T on it has finished
                        if (q_uses[s] > 0 && !mbar_wait(BAR(BAR_Q_EMPTY + s), (q_uses[s] - 1) & 1, p.err)) {
                            ok = false;
                            break;
                        }
                        const uint32_t dst = sQ0 + s * kTileBytes;
                        mbar_arrive_expect_tx(BAR(BAR_Q_FULL + s), kTileBytes);
                        tma_load_3d(dst, &tm_q, 0, w.hq0 + s, static_cast<int>(w.q0), BAR(BAR_Q_FULL + s));
                        tma_load_3d(dst + kBoxBytes, &tm_q, 64, w.hq0 + s, static_cast<int>(w.q0),
                                    BAR(BAR_Q_FULL + s));
                        ++q_uses[s];
                    }
                }
                ok = __shfl_sync(wmask, ok, 0);
                for (int k = 0; k < 2 * w.n_kv && ok; ++k, ++it) {   // K0, V0, K1, V1, ...
                    const uint32_t buf = it % kStages, use = it / kStages;
                    if (use > 0 && !mbar_wait(BAR(BAR_KV_EMPTY + buf), (use - 1) & 1, p.err)) ok = false;
                    if (!__all_sync(wmask, ok)) {
                        ok = false;
                        break;
                    }
                    const CUtensorMap *m = (k & 1) ? &tm_v : &tm_k;
                    const uint32_t dst = sKV0 + buf * kTileBytes;
                    const int row = static_cast<int>(w.kv0 + static_cast<long long>(k >> 1) * kBN);
                    // K_0 signals its own barrier; V_j and K_{j+1} both signal step barrier
                    // (gs + j) % 3, armed once for both when V_j is issued
                    const int j = (k - 1) >> 1;
                    const uint32_t bar = k == 0 ? BAR(BAR_K0_FULL) : BAR(BAR_STEP_FULL + (gs + j) % 3);
                    if (k == 0) {
                        if (lane == 0) mbar_arrive_expect_tx(bar, kTileBytes);
                        ++k0_uses;
                    } else if (k & 1) {
                        if (lane == 0) mbar_arrive_expect_tx(bar, j + 1 < w.n_kv ? 2 * kTileBytes : kTileBytes);
                        ++armed;
                    }
                    if (!paged) {
                        tma_load_3d(dst, m, 0, w.g, row, bar);
                        tma_load_3d(dst + kBoxBytes, m, 64, w.g, row, bar);
                    } else {
                        // a segment with no visible key, or behind a bad page id (reported
                        // once, with K), is read as zeros: a row past the pages' rows.  The
                        // boxes go out after lane 0 has armed the barrier.
                        __syncwarp();
                        if (seg_i < p.kv_segs) {
                            const int ps = p.kv_page_size;
                            int prow = p.kv_num_pages * ps;
                            if (row + seg_i * p.kv_seg_rows < kv_lim) {
                                if (pid_cur >= 0 && pid_cur < p.kv_num_pages) prow = pid_cur * ps + poff_cur;
                                else if (!(k & 1) && half == 0) atomicOr(p.err, kErrInput);
                            }
                            const uint32_t off = static_cast<uint32_t>(half) * kBoxBytes +
                                                 static_cast<uint32_t>(seg_i * p.kv_seg_rows) * 128u;
                            tma_load_3d(dst + off, m, 64 * half, w.g, prow, bar);
                        }
                        if (!(k & 1)) {   // K_j issued: fetch tile j+1's id while the ring turns
                            if ((k >> 1) + 1 < w.n_kv)
                                pid_nxt = kv_page_id(p, w.b, (k >> 1) + 1, kv_lim, seg_i, poff_nxt);
                        } else {
                            pid_cur = pid_nxt;
                            poff_cur = poff_nxt;
                        }
                    }
                }
                if (ok) gs += w.n_kv;
            }
            if (!ok && lane == 0) {
                // Failure path: let every copy still in flight land before the CTA exits.  No
                // barrier is re-armed before its previous phase completed, so waiting for the
                // last armed phase of each covers every copy (a step barrier armed for two
                // tiles of which only one was issued gives up after the bounded wait).
                for (int s = 0; s < 2; ++s)
                    if (q_uses[s] > 0) mbar_wait(BAR(BAR_Q_FULL + s), (q_uses[s] - 1) & 1, p.err);
                if (k0_uses > 0) mbar_wait(BAR(BAR_K0_FULL), (k0_uses - 1) & 1, p.err);
                for (int i = 0; i < 3; ++i) {
                    // steps 0 .. armed-1 were armed in order, so barrier i holds every third
                    const uint32_t arms = armed / 3 + (static_cast<uint32_t>(i) < armed % 3 ? 1u : 0u);
                    if (arms > 0) mbar_wait(BAR(BAR_STEP_FULL + i), (arms - 1) & 1, p.err);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // In-order program with blocking (suspending) waits, heads interleaved:
        //   per unit: Q K_0^T for each head as soon as its Q tile is ready; then for every
        //   tile j and head s: P_j V_j once the softmax has written P_j over S_j,
        //   immediately followed by Q K_{j+1}^T (which overwrites P_j: tcgen05.mma
        //   operations of one thread run in issue order).  While head 0's softmax works on
        //   S_{j+1}, the tensor core runs head 1's P V and Q K^T, and vice versa.  The
        //   first P V of a unit (accumulate off) waits until the epilogue has read O out.
        // The issuing thread is on the critical path: its queue of MMAs is shallow, so
        // every wait it makes idles the tensor core.  Its waits carry a short suspend hint
        // (a default try_wait can wake up ~900 cycles after the phase completes), and V_j
        // and K_{j+1} share one barrier so that each tile costs one wait for data.
#define MMA_WAIT(b_, par_) mbar_wait_hint((b_), (par_), 20u, p.err)
        if (lane == 0) {
            const uint32_t id_qk = idesc_bf16_f32(kBM, kBN, false);
            const uint32_t id_pv = idesc_bf16_f32(kBM, kHeadDim, true);
            bool ok = true;
            uint32_t q_uses[2] = {0u, 0u}, tiles[2] = {0u, 0u}, units[2] = {0u, 0u};
            uint32_t k0_uses = 0, it = 0, gs = 0;
            // failure-path test: a wait that nothing ends gives up after 100 us
            if (p.test_stall) ok = mbar_wait(BAR(BAR_NEVER), 0, p.err, 100000ull);
            for (int r = 0; ok; ++r) {
                const int u = attn_unit_of_round(r);
                if (u >= nun) break;
                AttnUnit w;
                bool bad;
                if (!attn_unit<LISTED>(p, u, w, bad)) continue;
                const uint32_t k0_item = it;
                if (!MMA_WAIT(BAR(BAR_K0_FULL), k0_uses & 1)) { ok = false; break; }
                ++k0_uses;
#pragma unroll
                for (int s = 0; s < 2; ++s) {   // unrolled: the per-head counters stay in registers
                    if (s >= w.nslots) break;
                    if (!MMA_WAIT(BAR(BAR_Q_READY + s), q_uses[s] & 1)) { ok = false; break; }
                    ++q_uses[s];
                    tc_fence_after();
                    issue_qk(tmem + s * 128, sQ0 + s * kTileBytes, sKV0 + (k0_item % kStages) * kTileBytes, id_qk);
                    umma_commit(BAR(BAR_S_FULL + s));
                    if (w.n_kv == 1) umma_commit(BAR(BAR_Q_EMPTY + s));
                }
                if (!ok) break;
                umma_commit(BAR(BAR_KV_EMPTY + k0_item % kStages));
                for (int j = 0; j < w.n_kv && ok; ++j) {
                    const uint32_t iv = k0_item + 2 * j + 1, ik = k0_item + 2 * j + 2;   // ring items of V_j, K_{j+1}
                    const bool more = j + 1 < w.n_kv;
                    if (!MMA_WAIT(BAR(BAR_STEP_FULL + (gs + j) % 3), ((gs + j) / 3) & 1)) { ok = false; break; }
#pragma unroll
                    for (int s = 0; s < 2; ++s) {
                        if (s >= w.nslots) break;
                        if (!MMA_WAIT(BAR(BAR_P_FULL + s), tiles[s] & 1)) { ok = false; break; }
                        ++tiles[s];
                        if (j == 0 && units[s] > 0 && !MMA_WAIT(BAR(BAR_O_EMPTY + s), (units[s] - 1) & 1)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_pv(tmem + 256 + s * 128, tmem + s * 128, sKV0 + (iv % kStages) * kTileBytes, id_pv, j > 0);
                        if (more) {
                            issue_qk(tmem + s * 128, sQ0 + s * kTileBytes, sKV0 + (ik % kStages) * kTileBytes, id_qk);
                            umma_commit(BAR(BAR_S_FULL + s));
                            if (j + 2 == w.n_kv) umma_commit(BAR(BAR_Q_EMPTY + s));
                        } else {
                            umma_commit(BAR(BAR_O_FULL + s));
                            ++units[s];
                        }
                    }
                    if (!ok) break;
                    umma_commit(BAR(BAR_KV_EMPTY + iv % kStages));
                    if (more) umma_commit(BAR(BAR_KV_EMPTY + ik % kStages));
                }
                it += 2 * w.n_kv;
                gs += w.n_kv;
            }
            // Every MMA issued above must finish before TMEM can be released.
            umma_commit(BAR(BAR_DRAIN));
            mbar_wait(BAR(BAR_DRAIN), 0, p.err);
        }
#undef MMA_WAIT
        __syncwarp();
    }
    } else {
        regs_inc<kRegsSoftmax>();
        // ------------------------------------------------------------ softmax warpgroups
        // Per unit: norm + rotate the Q tile, then the online softmax of every S tile.
        // The epilogue of a unit (O / l to global) runs after the next unit's Q tile has
        // been transformed, so that the next unit's first Q K^T overlaps it.
        const int s = (warp - 4) >> 2;
        const int r = tid - 128 * (1 + s);   // query row in the tile == TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + s * 128;
        const uint32_t tO = tmem + lane_base + 256 + s * 128;
        bool ok = true;
        uint32_t q_uses = 0, tiles = 0, units = 0;
        // the unit whose epilogue is pending: its query rows, their count and the head
        bool pend = false;
        float pend_l = 1.f;
        long long pend_q0 = 0;
        int pend_rows = 0, pend_hq = 0;
        const uint32_t stg = sbase + kOffStage + s * kStageBytes;   // this head's staging buffer
        const int wr = warp & 3;                                    // warp within the warpgroup
        int rnd = 0;
        while (ok) {
            AttnUnit w;
            bool have = false, bad;
            for (;; ++rnd) {
                const int u = attn_unit_of_round(rnd);
                if (u >= nun) break;
                if (attn_unit<LISTED>(p, u, w, bad) && s < w.nslots) {
                    have = true;
                    break;
                }
            }
            if (have) {
                ok = __all_sync(0xffffffffu, mbar_wait(BAR(BAR_Q_FULL + s), q_uses & 1, p.err));
                if (!ok) break;
                ++q_uses;
                const bool valid = r < w.rows;
                const long long tok = w.q0 + r;
                const int ps = valid ? p.pos[tok] : 0;
                transform_q_row<PAIRING>(sQ0 + s * kTileBytes, r, ps, valid ? p.rope_cs : nullptr, tok, p.wq, p.eps,
                                         p.rf);
                fence_proxy_async_smem();
                mbar_arrive(BAR(BAR_Q_READY + s));
            }
            if (pend) {
                ok = __all_sync(0xffffffffu, mbar_wait(BAR(BAR_O_FULL + s), units & 1, p.err));
                if (!ok) break;
                ++units;
                tc_fence_after();
                const float inv_l = 1.0f / pend_l;
                // O / l in four chunks of 32 columns: each thread stages its row (16-byte
                // granules swizzled by row, so that 8 consecutive rows hit distinct banks),
                // then its warp copies the warp's 32 rows out, 4 whole rows per instruction.
                // A warp reads back only rows it wrote, so a warp-level sync orders the two.
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    float o[32];
                    tmem_ld32(tO + 32 * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int g = 0; g < 8; ++g)
                        st_shared_v4(stg + r * 128 + ((g ^ (r & 7)) << 4),
                                     make_uint4(__float_as_uint(o[4 * g] * inv_l), __float_as_uint(o[4 * g + 1] * inv_l),
                                                __float_as_uint(o[4 * g + 2] * inv_l),
                                                __float_as_uint(o[4 * g + 3] * inv_l)));
                    __syncwarp();
                    const int g = lane & 7;
#pragma unroll
                    for (int it = 0; it < 8; ++it) {
                        const int row = wr * 32 + it * 4 + (lane >> 3);
                        const uint4 v = ld_shared_v4(stg + row * 128 + ((g ^ (row & 7)) << 4));
                        if (row < pend_rows) {
                            const long long e = ((pend_q0 + row) * p.H + pend_hq) * kHeadDim + 32 * c + 4 * g;
                            if (p.out_bf16)
                                *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(p.out) + e) =
                                    make_uint2(pack_bf16x2(__uint_as_float(v.x), __uint_as_float(v.y)),
                                               pack_bf16x2(__uint_as_float(v.z), __uint_as_float(v.w)));
                            else
                                *reinterpret_cast<uint4 *>(static_cast<float *>(p.out) + e) = v;
                        }
                    }
                    __syncwarp();   // the warp's rows of the staging buffer are free again
                }
                if (!ok) break;
                tc_fence_before();
                mbar_arrive(BAR(BAR_O_EMPTY + s));
                pend = false;
            }
            if (!have) break;

            // what the epilogue needs, copied now so that only n_kv and rowkey stay live
            const long long uq0 = w.q0;
            const int urows = w.rows, uhq = w.hq0 + s;
            const int n_kv = w.n_kv;
            const int rowkey = w.key0 + r;   // token index of this row: sees keys 0 .. rowkey
            float m_run = -INFINITY;   // running max of scaled scores (base 2), possibly stale by < 8
            float l_run = 0.f;         // running sum of 2^(score - m_run)
            for (int j = 0; j < n_kv && ok; ++j) {
                // S_FULL of tile j also means P_{j-1} V_{j-1} has finished (issued before Q K_j^T).
                ok = __all_sync(0xffffffffu, mbar_wait(BAR(BAR_S_FULL + s), tiles & 1, p.err));
                if (!ok) break;
                ++tiles;
                tc_fence_after();
                float x[128];
                tmem_ld32(tS, x);
                tmem_ld32(tS + 32, x + 32);
                tmem_ld32(tS + 64, x + 64);
                tmem_ld32(tS + 96, x + 96);
                tmem_wait_ld();
                const int lim = rowkey - j * kBN;   // keys c <= lim of this tile are visible
                if (lim < kBN - 1) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c > lim) x[c] = -INFINITY;
                }
                // The first tile sets the reference max from its own maximum (key 0 is visible
                // to every row, so it is finite).  Later tiles compute P against the current
                // reference straight away: a score more than 2^8 above it would make its own
                // term, and so the tile's sum, at least 2^8, so only a tile sum >= 250 calls
                // for the exact maximum and, if it grew by more than 2^8, a second pass.  The
                // reference, P and l are exactly those of finding the maximum first.
                if (j == 0) {
                    float m0[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) m0[e] = x[e];
#pragma unroll
                    for (int c = 8; c < 128; ++c) m0[c & 7] = fmaxf(m0[c & 7], x[c]);
                    m_run = max8(m0) * p.scale_log2;
                }
                float sp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                exp_tile(x, p.scale_log2, m_run == -INFINITY ? 0.f : -m_run, tS, sp);
                if (__any_sync(0xffffffffu, ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7])) >=
                                                250.0f || m_run == -INFINITY)) {
                    float mp[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) mp[e] = x[e];
#pragma unroll
                    for (int c = 8; c < 128; ++c) mp[c & 7] = fmaxf(mp[c & 7], x[c]);
                    const float m_new = fmaxf(m_run, max8(mp) * p.scale_log2);
                    // A row with no visible key yet (only past the end of its sequence) keeps
                    // -inf and adds nothing.
                    const bool need = m_new > m_run + 8.0f;
                    if (__any_sync(0xffffffffu, need)) {
                        // Move the reference, rescale l and this row of O (O is stable:
                        // P_{j-1} V_{j-1} finished before S_j was signalled), and write P again.
                        const float alpha = need ? ex2_approx(m_run - m_new) : 1.0f;
                        if (need) m_run = m_new;
                        l_run *= alpha;
                        if (need) {
#pragma unroll
                            for (int e = 0; e < 8; ++e) sp[e] = 0.f;
                        }
                        // lanes that keep their reference recompute the same P and sums
                        float sq[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                        exp_tile(x, p.scale_log2, m_run == -INFINITY ? 0.f : -m_run, tS, sq);
                        if (need) {
#pragma unroll
                            for (int e = 0; e < 8; ++e) sp[e] = sq[e];
                        }
#pragma unroll 1
                        for (int c = 0; c < 4; ++c) {
                            float o[32];
                            tmem_ld32(tO + 32 * c, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e) o[e] *= alpha;
                            tmem_st32(tO + 32 * c, o);
                        }
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(BAR(BAR_P_FULL + s));
                l_run += ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
            }
            pend = true;
            pend_l = l_run;
            pend_q0 = uq0;
            pend_rows = urows;
            pend_hq = uhq;
            ++rnd;
        }
        tc_fence_before();
    }
#undef BAR
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace gqa
