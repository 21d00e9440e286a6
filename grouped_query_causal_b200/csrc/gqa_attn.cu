// gqa_attn.cu -- host side of the C ABI declared in include/gqa_attn.h: argument
// validation, workspace carving, TMA tensor maps and kernel launches.  The kernels
// themselves live in prefill.cuh and decode.cuh (one translation unit, so no
// relocatable device code is needed).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "gqa_attn.h"
#include "decode.cuh"
#include "gemm.cuh"
#include "prefill.cuh"

namespace gqa {

// The device status word: error bits set by kernels (kErrTimeout, kErrInput).
__device__ unsigned g_device_error = 0;

namespace {

constexpr int kMaxDevices = 64;

// Failure-path test switch (gqa_attn_test_stall): read at every attention launch.
std::atomic<int> g_test_stall{0};

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    return dev;
}

// Device address of g_device_error on the current device (looked up once per device).
unsigned *device_error_word() {
    static std::atomic<unsigned *> cache[kMaxDevices];
    const int dev = current_device();
    if (dev < 0) return nullptr;
    unsigned *p = cache[dev].load(std::memory_order_acquire);
    if (p) return p;
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_device_error) != cudaSuccess) return nullptr;
    p = static_cast<unsigned *>(addr);
    cache[dev].store(p, std::memory_order_release);
    return p;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

// 3-D bf16 tensor [rows][heads][128] (head vectors contiguous, `row_bytes` between rows),
// box (64, 1, 128): half a head vector of 128 consecutive rows, 128-byte swizzle, zero
// fill outside the tensor.
bool make_rows_map(CUtensorMap *m, const void *base, uint64_t heads, uint64_t rows, uint64_t row_bytes,
                   uint32_t box_rows = 128) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), heads, rows};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDim) * 2, row_bytes};
    const cuuint32_t box[3] = {64, 1, box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

RopeFreqs rope_freqs(double theta) {
    RopeFreqs rf;
    for (int i = 0; i < kPairs; ++i) rf.inv_freq[i] = std::pow(theta, -2.0 * i / kHeadDim);
    return rf;
}

// The kernels' form of a RoPE variant, or false for an invalid configuration.
//   linear: theta_i / s;  ntk: (b s^(D/(D-2)))^(-2i/D);  yarn: with r_i = L theta_i / (2 pi)
//   and gamma_i = clamp((r_i - beta_slow) / (beta_fast - beta_slow), 0, 1),
//   theta_i ((1 - gamma_i) / s + gamma_i), and the logits times (0.1 ln s + 1)^2.
bool rope_spec(const gqa_rope_config *c, RopeSpec &out) {
    if (!c) return false;
    if (!(c->theta > 0.0) || !std::isfinite(c->theta)) return false;
    if (c->pairing != GQA_ROPE_PAIR_ADJACENT && c->pairing != GQA_ROPE_PAIR_HALF) return false;
    if (c->scaling < GQA_ROPE_SCALE_NONE || c->scaling > GQA_ROPE_SCALE_YARN) return false;
    const bool scaled = c->scaling != GQA_ROPE_SCALE_NONE;
    if (scaled && (!(c->factor >= 1.0) || !std::isfinite(c->factor))) return false;
    if (c->scaling == GQA_ROPE_SCALE_YARN &&
        (c->original_max_position < 1 || !std::isfinite(c->beta_fast) || !std::isfinite(c->beta_slow) ||
         !(c->beta_fast > c->beta_slow)))
        return false;
    const double s = scaled ? c->factor : 1.0;
    const double two_pi = 6.283185307179586476925286766559;
    const double ntk_base = c->theta * std::pow(s, static_cast<double>(kHeadDim) / (kHeadDim - 2));
    for (int i = 0; i < kPairs; ++i) {
        const double e = -2.0 * i / kHeadDim;
        double th = std::pow(c->theta, e);
        switch (c->scaling) {
            case GQA_ROPE_SCALE_LINEAR: th /= s; break;
            case GQA_ROPE_SCALE_NTK: th = std::pow(ntk_base, e); break;
            case GQA_ROPE_SCALE_YARN: {
                const double r = c->original_max_position * th / two_pi;
                const double gamma = std::min(1.0, std::max(0.0, (r - c->beta_slow) / (c->beta_fast - c->beta_slow)));
                th = (1.0 - gamma) * th / s + gamma * th;
                break;
            }
            default: break;
        }
        out.rf.inv_freq[i] = th;
    }
    out.pairing = c->pairing == GQA_ROPE_PAIR_HALF ? kPairHalf : kPairAdjacent;
    const double m = c->scaling == GQA_ROPE_SCALE_YARN ? 0.1 * std::log(s) + 1.0 : 1.0;
    out.logit_mult = static_cast<float>(m * m);
    return true;
}

// The plain RoPE of base theta (adjacent pairs, no scaling).
RopeSpec plain_rope(float theta) {
    RopeSpec r;
    r.rf = rope_freqs(static_cast<double>(theta));
    r.pairing = kPairAdjacent;
    r.logit_mult = 1.0f;
    return r;
}

int attn_sm_count() {
    static std::atomic<int> cache[kMaxDevices];
    const int dev = current_device();
    if (dev < 0) return 148;
    int n = cache[dev].load();
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev].store(n);
    return n;
}

bool attn_smem_attr_set() {
    static std::atomic<int> done[kMaxDevices];
    const int dev = current_device();
    if (dev < 0) return false;
    if (done[dev].load()) return true;
    const int bytes = static_cast<int>(kSmemBytes);
    const auto attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
    if (cudaFuncSetAttribute(attn_fwd_kernel<kPairAdjacent, false>, attr, bytes) != cudaSuccess ||
        cudaFuncSetAttribute(attn_fwd_kernel<kPairHalf, false>, attr, bytes) != cudaSuccess ||
        cudaFuncSetAttribute(attn_fwd_kernel<kPairAdjacent, true>, attr, bytes) != cudaSuccess ||
        cudaFuncSetAttribute(attn_fwd_kernel<kPairHalf, true>, attr, bytes) != cudaSuccess)
        return false;
    done[dev].store(1);
    return true;
}

bool prefill_shape_ok(int B, int T, int H, int Hkv) {
    if (B < 0 || T < 0 || H <= 0 || Hkv <= 0 || H % Hkv != 0) return false;
    // keep every element index and TMA extent well inside 64-bit / 32-bit limits
    if (static_cast<long long>(T) > (1LL << 30)) return false;
    const long long rows = static_cast<long long>(B) * T;
    if (rows > (1LL << 31)) return false;
    return true;
}

size_t decode_slots(int B, int H, int max_len) {
    const size_t maxC = (static_cast<size_t>(max_len) + kChunk - 1) / kChunk;
    return static_cast<size_t>(B) * maxC * static_cast<size_t>(H);
}

}  // namespace
}  // namespace gqa

using namespace gqa;

extern "C" const char *gqa_status_string(gqa_status status) {
    switch (status) {
        case GQA_OK: return "GQA_OK";
        case GQA_ERR_INVALID_ARG: return "GQA_ERR_INVALID_ARG";
        case GQA_ERR_UNSUPPORTED: return "GQA_ERR_UNSUPPORTED";
        case GQA_ERR_WORKSPACE: return "GQA_ERR_WORKSPACE";
        case GQA_ERR_CUDA: return "GQA_ERR_CUDA";
        case GQA_ERR_DEVICE_TIMEOUT: return "GQA_ERR_DEVICE_TIMEOUT";
        case GQA_ERR_DEVICE_INPUT: return "GQA_ERR_DEVICE_INPUT";
    }
    return "GQA_UNKNOWN_STATUS";
}

namespace {
// Workspace of gqa_attn_prefill: k-hat (bf16 [B,T,Hkv,D]), then the RoPE cos/sin table
// (round_up(B*T, 128) tokens x D fp32, blocked layout of rope_table_index).
size_t khat_bytes(int B, int T, int Hkv) { return round_up(static_cast<size_t>(B) * T * Hkv * kHeadDim * 2, 256); }
size_t rope_table_bytes(int B, int T) { return round_up(static_cast<size_t>(B) * T, 128) * kHeadDim * sizeof(float); }
// The unit list of a packed launch: at most one entry per 128 tokens of each sequence plus
// one per non-empty sequence (so at most N + N/128 + 1), then its count.
long long unit_list_entries(long long N) { return N + N / 128 + 1; }
size_t unit_list_bytes(long long N) { return round_up(static_cast<size_t>(unit_list_entries(N)) * 8, 256) + 256; }
}  // namespace

extern "C" size_t gqa_attn_prefill_workspace_size(int B, int T, int H, int Hkv, int D) {
    if (D != kHeadDim || !prefill_shape_ok(B, T, H, Hkv) || B == 0 || T == 0) return 0;
    return khat_bytes(B, T, Hkv) + rope_table_bytes(B, T);
}

namespace {

bool params_ok(float theta, float eps) {
    return theta > 0.f && std::isfinite(theta) && eps >= 0.f && std::isfinite(eps);
}

bool eps_ok(float eps) { return eps >= 0.f && std::isfinite(eps); }

// Where the k-hat prologue writes: row n (cu == nullptr), or, per sequence, after the
// rows already cached (the chunked-prefill append).
struct KRows {
    const int64_t *cu = nullptr, *cache_off = nullptr;
    const int32_t *prefix = nullptr;
    int B = 0;
    long long rows = 0;   // rows of the destination buffers
    const int32_t *pages = nullptr;   // paged destination (with cu): page table [B, max_pages]
    int page_size = 0, max_pages = 0, num_pages = 0;
};

// Enqueue the k-hat prologue (arguments already validated).  k rows are k_stride
// elements apart; v (optional) is copied beside k-hat into vout.
gqa_status launch_k_norm_rope(const void *k, long long k_stride, const void *v, long long v_stride, const int32_t *pos,
                              const float *knorm_w, const RopeSpec &rs, float eps, void *k_hat, void *vout,
                              float *rope_cs, long long ntok, int Hkv, const KRows &dst, cudaStream_t st) {
    unsigned *err = device_error_word();
    if (!err) return GQA_ERR_CUDA;
    KPrologueParams kp;
    kp.k = static_cast<const uint16_t *>(k);
    kp.v = static_cast<const uint16_t *>(v);
    kp.pos = pos;
    kp.wk = knorm_w;
    kp.khat = static_cast<uint16_t *>(k_hat);
    kp.vout = static_cast<uint16_t *>(vout);
    kp.rope_cs = rope_cs;
    kp.cu = dst.cu;
    kp.cache_off = dst.cache_off;
    kp.prefix = dst.prefix;
    kp.pages = dst.pages;
    kp.page_size = dst.page_size;
    kp.max_pages = dst.max_pages;
    kp.num_pages = dst.num_pages;
    kp.err = err;
    kp.ntok = ntok;
    kp.k_stride = k_stride;
    kp.v_stride = v_stride;
    kp.rows = dst.cu ? dst.rows : ntok;
    kp.Hkv = Hkv;
    kp.B = dst.B;
    kp.eps = eps;
    kp.rf = rs.rf;
    long long blocks = (ntok + 7) / 8;   // one warp per token, 8 warps per block
    const long long cap = static_cast<long long>(attn_sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    if (rs.pairing == kPairHalf)
        k_prologue_kernel<kPairHalf><<<static_cast<unsigned>(blocks), 256, 0, st>>>(kp);
    else
        k_prologue_kernel<kPairAdjacent><<<static_cast<unsigned>(blocks), 256, 0, st>>>(kp);
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

// Sequence geometry of an attention launch (AttnParams): dense (arrays null: B
// sequences of T tokens) or per sequence from device arrays.
struct AttnGeom {
    int B = 0, T = 0;                  // T: the dense length, or the longest sequence
    long long nq_rows = 0, nkv_rows = 0;
    long long q_row_elems = 0;         // elements between consecutive q rows (H*D unless strided)
    long long kv_row_elems = 0;        // elements between consecutive k-hat rows
    long long v_row_elems = 0;         // elements between consecutive v rows (0: as k-hat)
    bool out_bf16 = false;             // bf16 output (the input of the output projection)
    const int64_t *cu_q = nullptr, *kv_off = nullptr;
    const int32_t *prefix = nullptr;
    long long max_prefix = 0;          // host-side bound on the cached keys before a chunk (scheduling only)
    void *ulist_ws = nullptr;          // packed inputs: room for the unit list (unit_list_bytes of nq_rows)
    const int32_t *kv_pages = nullptr; // paged K/V: page table [B, kv_max_pages] (nkv_rows = kv_max_pages * kv_page_size)
    int kv_page_size = 0, kv_max_pages = 0, kv_num_pages = 0;
};

// Makespan, in 128-key tiles plus a fixed cost per unit (the next unit's Q transform and
// this unit's epilogue, about three tiles), of the dense units ordered band by band
// (`band` KV groups, latest query block first: attn_unit) and dealt to G persistent CTAs in
// snake order (attn_unit_of_round).  A dense unit of query block qb sweeps qb + 1 tiles.
long long dense_schedule_makespan(long long groups, int nqb, int npairs, long long band, int G) {
    constexpr long long kUnitOverheadTiles = 3;
    const long long per_band = band * nqb * npairs;
    const long long total = groups * nqb * npairs;
    std::vector<long long> cost(static_cast<size_t>(G), 0);
    for (long long r = 0; r * G < total; ++r)
        for (int c = 0; c < G; ++c) {
            const long long u = r * G + ((r & 1) ? G - 1 - c : c);
            if (u >= total) continue;
            const long long bi = u / per_band;
            const long long gb = std::min(band, groups - bi * band);
            const long long qb = nqb - 1 - (u - bi * per_band) / (gb * npairs);
            cost[static_cast<size_t>(c)] += qb + 1 + kUnitOverheadTiles;
        }
    return *std::max_element(cost.begin(), cost.end());
}

// KV groups (sequence, KV head) per band.  A band's K/V (the longest sequence's keys, K and
// V in bf16) should stay within ~80 MB of the 126 MB L2, which also carries Q, the output and
// the RoPE table, so that the CTAs working on a band re-read K/V from L2.  Bands are of equal
// size (the last one is not a short tail of long units).  Among the band sizes that fit, the
// band size also decides how evenly the snake order spreads the work over the CTAs, so for
// dense inputs, whose unit costs the host knows, the fewest bands are traded for up to four
// more when a simulation of the static schedule finishes earlier with them (decisions are
// kept per shape).  Packed inputs, whose lengths are on the device, are scheduled through the
// unit list instead (bands of whole sequences, launch_attention); without one they take the
// fewest bands.
int attn_band(const AttnGeom &gm, int Hkv, int nqb, int npairs, int G) {
    const long long groups = static_cast<long long>(gm.B) * Hkv;
    const long long keys = static_cast<long long>(gm.T) + gm.max_prefix;
    const long long kv_bytes = std::max(1LL, keys * kHeadDim * 2 * 2);
    const long long fit = std::max(1LL, (80LL << 20) / kv_bytes);
    const long long nb_min = (groups + fit - 1) / fit;
    const long long band0 = std::max(1LL, (groups + nb_min - 1) / nb_min);
    if (gm.cu_q != nullptr || nb_min == 1 || G <= 0 || groups * nqb * npairs > (1LL << 22))
        return static_cast<int>(band0);
    struct Entry {
        long long groups;
        int nqb, npairs, G;
        long long band0;
        int band;
    };
    static std::mutex mu;
    static std::vector<Entry> cache;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (const Entry &e : cache)
            if (e.groups == groups && e.nqb == nqb && e.npairs == npairs && e.G == G && e.band0 == band0)
                return e.band;
    }
    long long best = band0, best_span = dense_schedule_makespan(groups, nqb, npairs, band0, G);
    for (long long nb = nb_min + 1; nb <= std::min(groups, nb_min + 4); ++nb) {
        const long long b = (groups + nb - 1) / nb;
        if (b == best) continue;
        const long long span = dense_schedule_makespan(groups, nqb, npairs, b, G);
        if (span < best_span) {
            best = b;
            best_span = span;
        }
    }
    std::lock_guard<std::mutex> lock(mu);
    if (cache.size() >= 64) cache.erase(cache.begin());
    cache.push_back(Entry{groups, nqb, npairs, G, band0, static_cast<int>(best)});
    return static_cast<int>(best);
}

// Enqueue the attention kernel (arguments already validated); for packed inputs with room
// for a unit list, first the kernel that lists the units with work.
gqa_status launch_attention(const void *q, const void *k_hat, const void *v, const int32_t *pos,
                            const float *rope_cs, const float *qnorm_w, const RopeSpec &rs, float eps, void *out,
                            const AttnGeom &gm, int H, int Hkv, cudaStream_t st) {
    unsigned *err = device_error_word();
    if (!err) return GQA_ERR_CUDA;
    CUtensorMap tm_q, tm_k, tm_v;
    // paged K/V: the maps cover the pages' rows, one box per page segment of a tile
    const long long kv_map_rows =
        gm.kv_pages != nullptr ? static_cast<long long>(gm.kv_num_pages) * gm.kv_page_size : gm.nkv_rows;
    const uint32_t kv_box = gm.kv_pages != nullptr ? static_cast<uint32_t>(std::min(gm.kv_page_size, kBN)) : 128u;
    if (!make_rows_map(&tm_q, q, H, gm.nq_rows, gm.q_row_elems * 2) ||
        !make_rows_map(&tm_k, k_hat, Hkv, kv_map_rows, gm.kv_row_elems * 2, kv_box) ||
        !make_rows_map(&tm_v, v, Hkv, kv_map_rows, (gm.v_row_elems ? gm.v_row_elems : gm.kv_row_elems) * 2, kv_box))
        return GQA_ERR_CUDA;
    if (!attn_smem_attr_set()) return GQA_ERR_CUDA;
    AttnParams ap;
    ap.pos = pos;
    ap.rope_cs = rope_cs;
    ap.wq = qnorm_w;
    ap.out = out;
    ap.err = err;
    ap.cu_q = gm.cu_q;
    ap.kv_off = gm.kv_off;
    ap.prefix = gm.prefix;
    ap.kv_pages = gm.kv_pages;
    ap.kv_page_size = gm.kv_page_size;
    ap.kv_max_pages = gm.kv_max_pages;
    ap.kv_num_pages = gm.kv_num_pages;
    ap.kv_segs = gm.kv_page_size > 0 && gm.kv_page_size < kBN ? kBN / gm.kv_page_size : 1;
    ap.kv_seg_rows = kBN / ap.kv_segs;
    ap.nq_rows = gm.nq_rows;
    ap.nkv_rows = gm.nkv_rows;
    ap.B = gm.B;
    ap.T = gm.T;
    ap.H = H;
    ap.Hkv = Hkv;
    ap.hpg = H / Hkv;
    ap.nqb = (gm.T + kBM - 1) / kBM;
    ap.npairs = (ap.hpg + 1) / 2;
    ap.out_bf16 = gm.out_bf16 ? 1 : 0;
    ap.test_stall = g_test_stall.load(std::memory_order_relaxed);
    ap.eps = eps;
    ap.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kHeadDim))) * rs.logit_mult;
    ap.rf = rs.rf;
    const long long units = static_cast<long long>(ap.nqb) * gm.B * Hkv * ap.npairs;
    if (units <= 0) return GQA_OK;
    if (units > 0x7fffffffLL) return GQA_ERR_INVALID_ARG;
    ap.nunits = static_cast<int>(units);
    const unsigned grid = static_cast<unsigned>(std::min<long long>(units, attn_sm_count()));
    ap.ulist = nullptr;
    ap.ulist_n = nullptr;
    ap.uexp = Hkv * ap.npairs;
    const long long list_cap = unit_list_entries(gm.nq_rows);
    if (gm.cu_q != nullptr && gm.ulist_ws != nullptr && list_cap * ap.uexp <= 0x7fff0000LL) {
        // bands of sequences whose K/V (the longest sequence's keys) fit in ~80 MB of L2
        const long long seq_kv = std::max(1LL, (static_cast<long long>(gm.T) + gm.max_prefix) * Hkv * kHeadDim * 2 * 2);
        const long long fit = std::max(1LL, (80LL << 20) / seq_kv);
        const long long nb = (gm.B + fit - 1) / fit;
        const int band = static_cast<int>(std::max(1LL, (gm.B + nb - 1) / nb));
        int2 *list = static_cast<int2 *>(gm.ulist_ws);
        int *count = reinterpret_cast<int *>(static_cast<char *>(gm.ulist_ws) +
                                             round_up(static_cast<size_t>(list_cap) * 8, 256));
        unit_list_kernel<<<1, 1024, 0, st>>>(gm.cu_q, gm.kv_off, gm.prefix, gm.kv_pages != nullptr, gm.nq_rows,
                                             gm.nkv_rows, gm.B, ap.nqb, band, list, static_cast<int>(list_cap), count,
                                             err);
        if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
        ap.ulist = list;
        ap.ulist_n = count;
        ap.band = 1;
    } else {
        ap.band = attn_band(gm, Hkv, ap.nqb, ap.npairs, static_cast<int>(grid));
    }
    const bool listed = ap.ulist != nullptr;
    if (rs.pairing == kPairHalf) {
        if (listed)
            attn_fwd_kernel<kPairHalf, true><<<grid, kAttnThreads, kSmemBytes, st>>>(tm_q, tm_k, tm_v, ap);
        else
            attn_fwd_kernel<kPairHalf, false><<<grid, kAttnThreads, kSmemBytes, st>>>(tm_q, tm_k, tm_v, ap);
    } else {
        if (listed)
            attn_fwd_kernel<kPairAdjacent, true><<<grid, kAttnThreads, kSmemBytes, st>>>(tm_q, tm_k, tm_v, ap);
        else
            attn_fwd_kernel<kPairAdjacent, false><<<grid, kAttnThreads, kSmemBytes, st>>>(tm_q, tm_k, tm_v, ap);
    }
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

AttnGeom dense_geom(int B, int T, int H, int Hkv) {
    AttnGeom g;
    g.B = B;
    g.T = T;
    g.nq_rows = g.nkv_rows = static_cast<long long>(B) * T;
    g.q_row_elems = static_cast<long long>(H) * kHeadDim;
    g.kv_row_elems = static_cast<long long>(Hkv) * kHeadDim;
    return g;
}

}  // namespace

namespace {

gqa_status k_norm_rope_impl(const void *k, const int32_t *pos, const float *knorm_w, const RopeSpec &rs, float eps,
                            void *k_hat, float *rope_cs, int64_t N, int Hkv, int D, void *stream) {
    if (D != kHeadDim) return D > 0 ? GQA_ERR_UNSUPPORTED : GQA_ERR_INVALID_ARG;
    if (N < 0 || Hkv <= 0 || N > (1LL << 31)) return GQA_ERR_INVALID_ARG;
    if (N == 0) return GQA_OK;
    if (!k || !pos || !knorm_w || !k_hat) return GQA_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(k_hat, 16) || !aligned(knorm_w, 16) || !aligned(pos, 4) ||
        (rope_cs && !aligned(rope_cs, 16)))
        return GQA_ERR_INVALID_ARG;
    const size_t bytes = static_cast<size_t>(N) * Hkv * kHeadDim * 2;
    const uintptr_t a = reinterpret_cast<uintptr_t>(k), b = reinterpret_cast<uintptr_t>(k_hat);
    if (a < b + bytes && b < a + bytes) return GQA_ERR_INVALID_ARG;   // overlapping buffers
    if (rope_cs) {
        const uintptr_t c = reinterpret_cast<uintptr_t>(rope_cs);
        const size_t tb = round_up(static_cast<size_t>(N), 128) * kHeadDim * sizeof(float);
        if ((c < b + bytes && b < c + tb) || (c < a + bytes && a < c + tb)) return GQA_ERR_INVALID_ARG;
    }
    return launch_k_norm_rope(k, static_cast<long long>(Hkv) * kHeadDim, nullptr, 0, pos, knorm_w, rs, eps, k_hat,
                              nullptr, rope_cs, N, Hkv, KRows{}, static_cast<cudaStream_t>(stream));
}

gqa_status prefill_khat_impl(const void *q, const void *k_hat, const void *v, const int32_t *pos,
                             const float *rope_cs, const float *qnorm_w, const RopeSpec &rs, float eps, float *out,
                             int B, int T, int H, int Hkv, int D, void *stream) {
    if (D != kHeadDim) return D > 0 ? GQA_ERR_UNSUPPORTED : GQA_ERR_INVALID_ARG;
    if (!prefill_shape_ok(B, T, H, Hkv)) return GQA_ERR_INVALID_ARG;
    if (B == 0 || T == 0) return GQA_OK;
    if (!q || !k_hat || !v || !pos || !qnorm_w || !out) return GQA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_hat, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(qnorm_w, 16) ||
        !aligned(pos, 4) || (rope_cs && !aligned(rope_cs, 16)))
        return GQA_ERR_INVALID_ARG;
    return launch_attention(q, k_hat, v, pos, rope_cs, qnorm_w, rs, eps, out, dense_geom(B, T, H, Hkv), H, Hkv,
                            static_cast<cudaStream_t>(stream));
}

gqa_status prefill_impl(const void *q, const void *k, const void *v, const int32_t *pos, const float *qnorm_w,
                        const float *knorm_w, const RopeSpec &rs, float eps, float *out, int B, int T, int H,
                        int Hkv, int D, void *workspace, size_t workspace_bytes, void *stream) {
    if (D != kHeadDim) return D > 0 ? GQA_ERR_UNSUPPORTED : GQA_ERR_INVALID_ARG;
    if (!prefill_shape_ok(B, T, H, Hkv)) return GQA_ERR_INVALID_ARG;
    if (B == 0 || T == 0) return GQA_OK;
    if (!q || !k || !v || !pos || !qnorm_w || !knorm_w || !out) return GQA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(qnorm_w, 16) ||
        !aligned(knorm_w, 16) || !aligned(pos, 4))
        return GQA_ERR_INVALID_ARG;
    const size_t need = gqa_attn_prefill_workspace_size(B, T, H, Hkv, D);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return GQA_ERR_WORKSPACE;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *table = reinterpret_cast<float *>(static_cast<char *>(workspace) + khat_bytes(B, T, Hkv));
    gqa_status s = launch_k_norm_rope(k, static_cast<long long>(Hkv) * kHeadDim, nullptr, 0, pos, knorm_w, rs, eps,
                                      workspace, nullptr, table, static_cast<long long>(B) * T, Hkv, KRows{}, st);
    if (s != GQA_OK) return s;
    return launch_attention(q, workspace, v, pos, table, qnorm_w, rs, eps, out, dense_geom(B, T, H, Hkv), H, Hkv,
                            st);
}

}  // namespace

extern "C" gqa_status gqa_attn_k_norm_rope(const void *k, const int32_t *pos, const float *knorm_w, float theta,
                                           float eps, void *k_hat, float *rope_cs, int64_t N, int Hkv, int D,
                                           void *stream) {
    if (!params_ok(theta, eps)) return GQA_ERR_INVALID_ARG;
    return k_norm_rope_impl(k, pos, knorm_w, plain_rope(theta), eps, k_hat, rope_cs, N, Hkv, D, stream);
}

extern "C" gqa_status gqa_attn_k_norm_rope_ex(const void *k, const int32_t *pos, const float *knorm_w,
                                              const gqa_rope_config *rope, float eps, void *k_hat, float *rope_cs,
                                              int64_t N, int Hkv, int D, void *stream) {
    RopeSpec rs;
    if (!rope_spec(rope, rs) || !eps_ok(eps)) return GQA_ERR_INVALID_ARG;
    return k_norm_rope_impl(k, pos, knorm_w, rs, eps, k_hat, rope_cs, N, Hkv, D, stream);
}

extern "C" gqa_status gqa_attn_prefill_khat(const void *q, const void *k_hat, const void *v, const int32_t *pos,
                                            const float *rope_cs, const float *qnorm_w, float theta, float eps,
                                            float *out, int B, int T, int H, int Hkv, int D, void *stream) {
    if (!params_ok(theta, eps)) return GQA_ERR_INVALID_ARG;
    return prefill_khat_impl(q, k_hat, v, pos, rope_cs, qnorm_w, plain_rope(theta), eps, out, B, T, H, Hkv, D,
                             stream);
}

extern "C" gqa_status gqa_attn_prefill_khat_ex(const void *q, const void *k_hat, const void *v, const int32_t *pos,
                                               const float *rope_cs, const float *qnorm_w,
                                               const gqa_rope_config *rope, float eps, float *out, int B, int T,
                                               int H, int Hkv, int D, void *stream) {
    RopeSpec rs;
    if (!rope_spec(rope, rs) || !eps_ok(eps)) return GQA_ERR_INVALID_ARG;
    return prefill_khat_impl(q, k_hat, v, pos, rope_cs, qnorm_w, rs, eps, out, B, T, H, Hkv, D, stream);
}

extern "C" gqa_status gqa_attn_prefill(const void *q, const void *k, const void *v, const int32_t *pos,
                                       const float *qnorm_w, const float *knorm_w, float theta, float eps,
                                       float *out, int B, int T, int H, int Hkv, int D, void *workspace,
                                       size_t workspace_bytes, void *stream) {
    if (!params_ok(theta, eps)) return GQA_ERR_INVALID_ARG;
    return prefill_impl(q, k, v, pos, qnorm_w, knorm_w, plain_rope(theta), eps, out, B, T, H, Hkv, D, workspace,
                        workspace_bytes, stream);
}

extern "C" gqa_status gqa_attn_prefill_ex(const void *q, const void *k, const void *v, const int32_t *pos,
                                          const float *qnorm_w, const float *knorm_w, const gqa_rope_config *rope,
                                          float eps, float *out, int B, int T, int H, int Hkv, int D,
                                          void *workspace, size_t workspace_bytes, void *stream) {
    RopeSpec rs;
    if (!rope_spec(rope, rs) || !eps_ok(eps)) return GQA_ERR_INVALID_ARG;
    return prefill_impl(q, k, v, pos, qnorm_w, knorm_w, rs, eps, out, B, T, H, Hkv, D, workspace, workspace_bytes,
                        stream);
}

// ---------------------------------------------------------------- packed and chunked prefill
namespace {

bool ragged_shape_ok(int B, int64_t N, int H, int Hkv, int max_len) {
    if (B < 0 || N < 0 || H <= 0 || Hkv <= 0 || H % Hkv != 0 || max_len < 0) return false;
    if (N > (1LL << 31) - 256 || max_len > (1 << 30)) return false;
    return true;
}

}  // namespace

extern "C" size_t gqa_attn_prefill_varlen_workspace_size(int64_t N, int Hkv, int D) {
    if (D != kHeadDim || N <= 0 || Hkv <= 0 || N > (1LL << 31) - 256) return 0;
    return khat_bytes(1, static_cast<int>(N), Hkv) + rope_table_bytes(1, static_cast<int>(N)) + unit_list_bytes(N);
}

extern "C" gqa_status gqa_attn_prefill_varlen(const void *q, const void *k, const void *v, const int32_t *pos,
                                              const int64_t *cu_seqlens, const float *qnorm_w, const float *knorm_w,
                                              const gqa_rope_config *rope, float eps, float *out, int B, int64_t N,
                                              int H, int Hkv, int D, int max_seqlen, void *workspace,
                                              size_t workspace_bytes, void *stream) {
    RopeSpec rs;
    if (!rope_spec(rope, rs) || !eps_ok(eps)) return GQA_ERR_INVALID_ARG;
    if (D != kHeadDim) return D > 0 ? GQA_ERR_UNSUPPORTED : GQA_ERR_INVALID_ARG;
    if (!ragged_shape_ok(B, N, H, Hkv, max_seqlen)) return GQA_ERR_INVALID_ARG;
    if (B == 0 || N == 0 || max_seqlen == 0) return GQA_OK;
    if (!q || !k || !v || !pos || !cu_seqlens || !qnorm_w || !knorm_w || !out) return GQA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(qnorm_w, 16) ||
        !aligned(knorm_w, 16) || !aligned(pos, 4) || !aligned(cu_seqlens, 8))
        return GQA_ERR_INVALID_ARG;
    const size_t need = gqa_attn_prefill_varlen_workspace_size(N, Hkv, D);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return GQA_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void *khat = workspace;
    float *table = reinterpret_cast<float *>(static_cast<char *>(workspace) + khat_bytes(1, static_cast<int>(N), Hkv));
    gqa_status s = launch_k_norm_rope(k, static_cast<long long>(Hkv) * kHeadDim, nullptr, 0, pos, knorm_w, rs, eps,
                                      khat, nullptr, table, N, Hkv, KRows{}, st);
    if (s != GQA_OK) return s;
    AttnGeom gm;
    gm.B = B;
    gm.T = max_seqlen;
    gm.nq_rows = gm.nkv_rows = N;
    gm.q_row_elems = static_cast<long long>(H) * kHeadDim;
    gm.kv_row_elems = static_cast<long long>(Hkv) * kHeadDim;
    gm.cu_q = cu_seqlens;
    gm.ulist_ws = reinterpret_cast<char *>(table) + rope_table_bytes(1, static_cast<int>(N));
    return launch_attention(q, khat, v, pos, table, qnorm_w, rs, eps, out, gm, H, Hkv, st);
}

extern "C" size_t gqa_attn_prefill_chunk_workspace_size(int64_t N, int D) {
    if (D != kHeadDim || N <= 0 || N > (1LL << 31) - 256) return 0;
    return rope_table_bytes(1, static_cast<int>(N)) + unit_list_bytes(N);
}

extern "C" gqa_status gqa_attn_prefill_chunk(const void *q, const void *k, const void *v, const int32_t *pos,
                                             const int64_t *cu_seqlens, void *k_cache, void *v_cache,
                                             const int64_t *cache_offsets, const int32_t *prefix_len,
                                             int64_t cache_rows, const float *qnorm_w, const float *knorm_w,
                                             const gqa_rope_config *rope, float eps, float *out, int B, int64_t N,
                                             int H, int Hkv, int D, int max_chunk_len, void *workspace,
                                             size_t workspace_bytes, void *stream) {
    RopeSpec rs;
    if (!rope_spec(rope, rs) || !eps_ok(eps)) return GQA_ERR_INVALID_ARG;
    if (D != kHeadDim) return D > 0 ? GQA_ERR_UNSUPPORTED : GQA_ERR_INVALID_ARG;
    if (!ragged_shape_ok(B, N, H, Hkv, max_chunk_len)) return GQA_ERR_INVALID_ARG;
    if (cache_rows < 0 || cache_rows > (1LL << 31) - 256) return GQA_ERR_INVALID_ARG;
    if (B == 0 || N == 0 || max_chunk_len == 0) return GQA_OK;
    if (!q || !k || !v || !pos || !cu_seqlens || !k_cache || !v_cache || !cache_offsets || !prefix_len ||
        !qnorm_w || !knorm_w || !out || cache_rows == 0)
        return GQA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(qnorm_w, 16) ||
        !aligned(knorm_w, 16) || !aligned(pos, 4) || !aligned(cu_seqlens, 8) || !aligned(k_cache, 16) ||
        !aligned(v_cache, 16) || !aligned(cache_offsets, 8) || !aligned(prefix_len, 4))
        return GQA_ERR_INVALID_ARG;
    const size_t need = gqa_attn_prefill_chunk_workspace_size(N, D);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return GQA_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *table = static_cast<float *>(workspace);
    // the chunk's k-hat and v go into the cache after each sequence's cached rows ...
    KRows dst;
    dst.cu = cu_seqlens;
    dst.cache_off = cache_offsets;
    dst.prefix = prefix_len;
    dst.B = B;
    dst.rows = cache_rows;
    const long long kv = static_cast<long long>(Hkv) * kHeadDim;
    gqa_status s = launch_k_norm_rope(k, kv, v, kv, pos, knorm_w, rs, eps, k_cache, v_cache, table, N, Hkv, dst, st);
    if (s != GQA_OK) return s;
    // ... and the chunk's queries attend to all of them
    AttnGeom gm;
    gm.B = B;
    gm.T = max_chunk_len;
    gm.nq_rows = N;
    gm.nkv_rows = cache_rows;
    gm.q_row_elems = static_cast<long long>(H) * kHeadDim;
    gm.kv_row_elems = kv;
    gm.cu_q = cu_seqlens;
    gm.kv_off = cache_offsets;
    gm.prefix = prefix_len;
    gm.max_prefix = cache_rows / std::max(1, B);   // an average; only the schedule depends on it
    gm.ulist_ws = reinterpret_cast<char *>(table) + rope_table_bytes(1, static_cast<int>(N));
    return launch_attention(q, k_cache, v_cache, pos, table, qnorm_w, rs, eps, out, gm, H, Hkv, st);
}

extern "C" size_t gqa_attn_prefill_chunk_paged_workspace_size(int64_t N, int D) {
    return gqa_attn_prefill_chunk_workspace_size(N, D);
}

extern "C" gqa_status gqa_attn_prefill_chunk_paged(const void *q, const void *k, const void *v, const int32_t *pos,
                                                   const int64_t *cu_seqlens, void *k_pages, void *v_pages,
                                                   const int32_t *page_table, int num_pages, int page_size,
                                                   int max_pages, const int32_t *prefix_len, const float *qnorm_w,
                                                   const float *knorm_w, const gqa_rope_config *rope, float eps,
                                                   float *out, int B, int64_t N, int H, int Hkv, int D,
                                                   int max_chunk_len, void *workspace, size_t workspace_bytes,
                                                   void *stream) {
    RopeSpec rs;
    if (!rope_spec(rope, rs) || !eps_ok(eps)) return GQA_ERR_INVALID_ARG;
    if (D != kHeadDim) return D > 0 ? GQA_ERR_UNSUPPORTED : GQA_ERR_INVALID_ARG;
    if (!ragged_shape_ok(B, N, H, Hkv, max_chunk_len)) return GQA_ERR_INVALID_ARG;
    if (num_pages <= 0 || max_pages <= 0 || page_size <= 0 || page_size % 16 != 0) return GQA_ERR_INVALID_ARG;
    // a 128-key tile must be whole pages or lie inside one page
    if (kBN % page_size != 0 && page_size % kBN != 0) return GQA_ERR_UNSUPPORTED;
    if (static_cast<long long>(num_pages) * page_size > (1LL << 31) - 256 ||
        static_cast<long long>(max_pages) * page_size > (1LL << 31) - 256)
        return GQA_ERR_INVALID_ARG;
    if (B == 0 || N == 0 || max_chunk_len == 0) return GQA_OK;
    if (!q || !k || !v || !pos || !cu_seqlens || !k_pages || !v_pages || !page_table || !prefix_len || !qnorm_w ||
        !knorm_w || !out)
        return GQA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(qnorm_w, 16) ||
        !aligned(knorm_w, 16) || !aligned(pos, 4) || !aligned(cu_seqlens, 8) || !aligned(k_pages, 16) ||
        !aligned(v_pages, 16) || !aligned(page_table, 4) || !aligned(prefix_len, 4))
        return GQA_ERR_INVALID_ARG;
    const size_t need = gqa_attn_prefill_chunk_paged_workspace_size(N, D);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return GQA_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float *table = static_cast<float *>(workspace);
    // the chunk's k-hat and v go into the pages after each sequence's cached rows ...
    KRows dst;
    dst.cu = cu_seqlens;
    dst.prefix = prefix_len;
    dst.B = B;
    dst.rows = static_cast<long long>(num_pages) * page_size;
    dst.pages = page_table;
    dst.page_size = page_size;
    dst.max_pages = max_pages;
    dst.num_pages = num_pages;
    const long long kv = static_cast<long long>(Hkv) * kHeadDim;
    gqa_status s = launch_k_norm_rope(k, kv, v, kv, pos, knorm_w, rs, eps, k_pages, v_pages, table, N, Hkv, dst, st);
    if (s != GQA_OK) return s;
    // ... and the chunk's queries attend to all of them through the page table
    AttnGeom gm;
    gm.B = B;
    gm.T = max_chunk_len;
    gm.nq_rows = N;
    gm.nkv_rows = static_cast<long long>(max_pages) * page_size;
    gm.q_row_elems = static_cast<long long>(H) * kHeadDim;
    gm.kv_row_elems = kv;
    gm.cu_q = cu_seqlens;
    gm.prefix = prefix_len;
    gm.max_prefix = static_cast<long long>(num_pages) * page_size / std::max(1, B);   // scheduling only
    gm.ulist_ws = reinterpret_cast<char *>(table) + rope_table_bytes(1, static_cast<int>(N));
    gm.kv_pages = page_table;
    gm.kv_page_size = page_size;
    gm.kv_max_pages = max_pages;
    gm.kv_num_pages = num_pages;
    return launch_attention(q, k_pages, v_pages, pos, table, qnorm_w, rs, eps, out, gm, H, Hkv, st);
}

// ---------------------------------------------------------------- projections
namespace {

// 2-D bf16 matrix [rows][cols] (row stride ld elements), box (64 cols, box_rows rows),
// 128-byte swizzle, zero fill outside.
bool make_matrix_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {ld * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool gemm_smem_attr_set() {
    static std::atomic<int> done[kMaxDevices];
    const int dev = current_device();
    if (dev < 0) return false;
    if (done[dev].load()) return true;
    if (cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kGemmSmemBytes)) != cudaSuccess)
        return false;
    done[dev].store(1);
    return true;
}

// y[M, N] = x[M, K] w[N, K]^T (arguments validated): x rows ldx elements apart, y rows ldy.
gqa_status launch_gemm(const void *x, long long ldx, const void *w, void *y, long long ldy, bool y_fp32, int M, int N,
                       int K, cudaStream_t st) {
    unsigned *err = device_error_word();
    if (!err) return GQA_ERR_CUDA;
    CUtensorMap tm_x, tm_w;
    if (!make_matrix_map(&tm_x, x, M, K, ldx, kGemmBM) || !make_matrix_map(&tm_w, w, N, K, K, kGemmBN))
        return GQA_ERR_CUDA;
    if (!gemm_smem_attr_set()) return GQA_ERR_CUDA;
    GemmParams gp;
    gp.y = y;
    gp.err = err;
    gp.M = M;
    gp.N = N;
    gp.K = K;
    gp.ldy = ldy;
    gp.y_fp32 = y_fp32 ? 1 : 0;
    gp.mblocks = (M + kGemmBM - 1) / kGemmBM;
    gp.nblocks = (N + kGemmBN - 1) / kGemmBN;
    const long long tiles = static_cast<long long>(gp.mblocks) * gp.nblocks;
    if (tiles <= 0) return GQA_OK;
    if (tiles > 0x7fffffffLL) return GQA_ERR_INVALID_ARG;
    gp.ntiles = static_cast<int>(tiles);
    const unsigned grid = static_cast<unsigned>(std::min<long long>(tiles, attn_sm_count()));
    gemm_kernel<<<grid, kGemmThreads, kGemmSmemBytes, st>>>(tm_x, tm_w, gp);
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

bool linear_shape_ok(long long M, long long N, long long K) {
    return M >= 0 && N > 0 && K > 0 && N % 32 == 0 && K % 8 == 0 && M < (1LL << 31) && N < (1LL << 24) &&
           K < (1LL << 24);
}

}  // namespace

extern "C" gqa_status gqa_linear(const void *x, const void *w, void *y, int y_dtype, int64_t M, int N, int K,
                                 void *stream) {
    if (y_dtype != GQA_DTYPE_BF16 && y_dtype != GQA_DTYPE_F32) return GQA_ERR_INVALID_ARG;
    if (!linear_shape_ok(M, N, K)) return GQA_ERR_INVALID_ARG;
    if (M == 0) return GQA_OK;
    if (!x || !w || !y || !aligned(x, 16) || !aligned(w, 16) || !aligned(y, 16)) return GQA_ERR_INVALID_ARG;
    return launch_gemm(x, K, w, y, N, y_dtype == GQA_DTYPE_F32, static_cast<int>(M), N, K,
                       static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- the whole attention sub-block
namespace {

struct BlockLayout {
    size_t qkv, khat, table, o, total;
};

bool block_layout(int B, int T, int H, int Hkv, BlockLayout &l) {
    if (!prefill_shape_ok(B, T, H, Hkv) || B == 0 || T == 0) return false;
    const size_t n = static_cast<size_t>(B) * T;
    l.qkv = 0;
    l.khat = round_up(n * (H + 2 * Hkv) * kHeadDim * 2, 256);
    l.table = l.khat + khat_bytes(B, T, Hkv);
    l.o = l.table + rope_table_bytes(B, T);
    l.total = l.o + round_up(n * H * kHeadDim * 2, 256);
    return true;
}

}  // namespace

extern "C" size_t gqa_attn_block_prefill_workspace_size(int B, int T, int hidden, int H, int Hkv, int D) {
    BlockLayout l;
    if (D != kHeadDim || hidden <= 0 || !block_layout(B, T, H, Hkv, l)) return 0;
    return l.total;
}

extern "C" gqa_status gqa_attn_block_prefill(const void *x, const void *w_qkv, const void *w_o, const int32_t *pos,
                                             const float *qnorm_w, const float *knorm_w, const gqa_rope_config *rope,
                                             float eps, float *y, int B, int T, int hidden, int H, int Hkv, int D,
                                             void *workspace, size_t workspace_bytes, void *stream) {
    RopeSpec rs;
    if (!rope_spec(rope, rs) || !eps_ok(eps)) return GQA_ERR_INVALID_ARG;
    if (D != kHeadDim) return D > 0 ? GQA_ERR_UNSUPPORTED : GQA_ERR_INVALID_ARG;
    if (!prefill_shape_ok(B, T, H, Hkv)) return GQA_ERR_INVALID_ARG;
    const long long n = static_cast<long long>(B) * T;
    const int nqkv = (H + 2 * Hkv) * kHeadDim;
    if (hidden <= 0 || !linear_shape_ok(n, nqkv, hidden) || !linear_shape_ok(n, hidden, H * kHeadDim))
        return GQA_ERR_INVALID_ARG;
    if (n == 0) return GQA_OK;
    if (!x || !w_qkv || !w_o || !pos || !qnorm_w || !knorm_w || !y) return GQA_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w_qkv, 16) || !aligned(w_o, 16) || !aligned(y, 16) || !aligned(qnorm_w, 16) ||
        !aligned(knorm_w, 16) || !aligned(pos, 4))
        return GQA_ERR_INVALID_ARG;
    BlockLayout l;
    if (!block_layout(B, T, H, Hkv, l)) return GQA_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < l.total) return GQA_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);
    uint16_t *qkv = reinterpret_cast<uint16_t *>(ws + l.qkv);
    void *khat = ws + l.khat;
    float *table = reinterpret_cast<float *>(ws + l.table);
    void *o = ws + l.o;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // (1) qkv = x W_qkv^T, bf16 [n, H + 2 Hkv, D]: q, k, v of a token side by side
    gqa_status s = launch_gemm(x, hidden, w_qkv, qkv, nqkv, false, static_cast<int>(n), nqkv, hidden, st);
    if (s != GQA_OK) return s;
    // (2) k-hat from the k section, read in place
    s = launch_k_norm_rope(qkv + static_cast<size_t>(H) * kHeadDim, nqkv, nullptr, 0, pos, knorm_w, rs, eps, khat,
                           nullptr, table, n, Hkv, KRows{}, st);
    if (s != GQA_OK) return s;
    // (3) attention on the q and v sections in place, bf16 output [n, H, D]
    AttnGeom gm = dense_geom(B, T, H, Hkv);
    gm.q_row_elems = nqkv;
    gm.v_row_elems = nqkv;
    gm.out_bf16 = true;
    s = launch_attention(qkv, khat, qkv + static_cast<size_t>(H + Hkv) * kHeadDim, pos, table, qnorm_w, rs, eps, o, gm,
                         H, Hkv, st);
    if (s != GQA_OK) return s;
    // (4) y = o W_o^T over the concatenated heads, fp32 [n, hidden]
    return launch_gemm(o, static_cast<long long>(H) * kHeadDim, w_o, y, hidden, true, static_cast<int>(n), hidden,
                       H * kHeadDim, st);
}

extern "C" size_t gqa_attn_decode_workspace_size(int B, int H, int Hkv, int D, int max_len) {
    if (B <= 0 || H <= 0 || Hkv <= 0 || H % Hkv != 0 || D != kHeadDim || max_len <= 0) return 0;
    const size_t slots = decode_slots(B, H, max_len);
    return round_up(slots * kHeadDim * sizeof(float), 256) + round_up(slots * 2 * sizeof(float), 256);
}

namespace {
template <int HG>
gqa_status launch_decode(const DecodeParams &p, int npass, cudaStream_t st) {
    const dim3 grid(static_cast<unsigned>(p.B * p.Hkv), static_cast<unsigned>(p.maxC), static_cast<unsigned>(npass));
    if (p.pages != nullptr)
        decode_split_kernel<HG, true><<<grid, 128, 0, st>>>(p);
    else
        decode_split_kernel<HG, false><<<grid, 128, 0, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
    decode_merge_kernel<<<static_cast<unsigned>(p.B * p.H), 128, 0, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
    return GQA_OK;
}
}  // namespace

namespace {

// Shared body of the decode entry points.  With k_new != nullptr the new token is first
// appended to the cache (decode_append_kernel) and the split kernel attends to one row
// more than seqlens[b].
// A paged cache: page table [B, max_pages] of page ids < num_pages, page_size rows a page.
struct PagedCache {
    const int32_t *pages;
    int num_pages, page_size, max_pages;
};

// Host-side argument checks of the decode entry points, everything except the
// workspace.  Sets `empty` for B == 0 (a no-op).
gqa_status decode_check(const void *q, const void *k_new, const void *v_new, const void *k_cache,
                        const void *v_cache, const int64_t *cache_offsets, const PagedCache *paged,
                        const int32_t *seqlens, const int32_t *q_pos, const float *qnorm_w, const float *knorm_w,
                        float eps, const float *out, int B, int H, int Hkv, int D, int max_len, bool &empty) {
    empty = false;
    const bool append = k_new != nullptr || v_new != nullptr || knorm_w != nullptr;
    if (D != kHeadDim) return D > 0 ? GQA_ERR_UNSUPPORTED : GQA_ERR_INVALID_ARG;
    if (B < 0 || H <= 0 || Hkv <= 0 || H % Hkv != 0) return GQA_ERR_INVALID_ARG;
    if (!eps_ok(eps)) return GQA_ERR_INVALID_ARG;
    if (B == 0) {
        empty = true;
        return GQA_OK;
    }
    if (max_len <= 0) return GQA_ERR_INVALID_ARG;
    if ((static_cast<long long>(max_len) + kChunk - 1) / kChunk > 65535) return GQA_ERR_INVALID_ARG;
    if (static_cast<long long>(B) * Hkv > 0x7fffffffLL || static_cast<long long>(B) * H > 0x7fffffffLL)
        return GQA_ERR_INVALID_ARG;
    if (!q || !k_cache || !v_cache || !seqlens || !qnorm_w || !out) return GQA_ERR_INVALID_ARG;
    if (paged) {
        if (!paged->pages || !aligned(paged->pages, 4) || paged->num_pages < 1 || paged->max_pages < 1 ||
            paged->page_size < 16 || paged->page_size % 16 != 0 ||
            static_cast<long long>(B) * paged->max_pages > 0x7fffffffLL)
            return GQA_ERR_INVALID_ARG;
    } else if (!cache_offsets || !aligned(cache_offsets, 8)) {
        return GQA_ERR_INVALID_ARG;
    }
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(qnorm_w, 16) ||
        !aligned(out, 4) || !aligned(seqlens, 4) || (q_pos && !aligned(q_pos, 4)))
        return GQA_ERR_INVALID_ARG;
    if (append && (!k_new || !v_new || !knorm_w || !aligned(k_new, 8) || !aligned(v_new, 8) || !aligned(knorm_w, 16)))
        return GQA_ERR_INVALID_ARG;
    return GQA_OK;
}

gqa_status decode_impl(const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                       const int64_t *cache_offsets, const PagedCache *paged, const int32_t *seqlens,
                       const int32_t *q_pos,
                       const float *qnorm_w, const float *knorm_w, const RopeSpec &rs, float eps, float *out, int B,
                       int H, int Hkv, int D, int max_len, void *workspace, size_t workspace_bytes, void *stream) {
    const bool append = k_new != nullptr || v_new != nullptr || knorm_w != nullptr;
    bool empty = false;
    const gqa_status chk = decode_check(q, k_new, v_new, k_cache, v_cache, cache_offsets, paged, seqlens, q_pos,
                                        qnorm_w, knorm_w, eps, out, B, H, Hkv, D, max_len, empty);
    if (chk != GQA_OK || empty) return chk;
    const size_t need = gqa_attn_decode_workspace_size(B, H, Hkv, D, max_len);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return GQA_ERR_WORKSPACE;
    unsigned *err = device_error_word();
    if (!err) return GQA_ERR_CUDA;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (append) {
        AppendParams ap;
        ap.k_new = static_cast<const uint16_t *>(k_new);
        ap.v_new = static_cast<const uint16_t *>(v_new);
        ap.kc = static_cast<uint16_t *>(k_cache);
        ap.vc = static_cast<uint16_t *>(v_cache);
        ap.offsets = cache_offsets;
        ap.seqlens = seqlens;
        ap.qpos = q_pos;
        ap.wk = knorm_w;
        ap.err = err;
        ap.B = B;
        ap.Hkv = Hkv;
        ap.max_len = max_len;
        ap.pairing = rs.pairing;
        ap.pages = paged ? paged->pages : nullptr;
        ap.page_size = paged ? paged->page_size : 0;
        ap.max_pages = paged ? paged->max_pages : 0;
        ap.num_pages = paged ? paged->num_pages : 0;
        ap.eps = eps;
        ap.rf = rs.rf;
        const long long warps = static_cast<long long>(B) * Hkv;
        decode_append_kernel<<<static_cast<unsigned>((warps + 3) / 4), 128, 0, st>>>(ap);
        if (cudaGetLastError() != cudaSuccess) return GQA_ERR_CUDA;
    }

    const size_t slots = decode_slots(B, H, max_len);
    DecodeParams p;
    p.q = static_cast<const uint16_t *>(q);
    p.kc = static_cast<const uint16_t *>(k_cache);
    p.vc = static_cast<const uint16_t *>(v_cache);
    p.offsets = cache_offsets;
    p.seqlens = seqlens;
    p.qpos = q_pos;
    p.wq = qnorm_w;
    p.part_o = static_cast<float *>(workspace);
    p.part_ml = reinterpret_cast<float *>(static_cast<char *>(workspace) + round_up(slots * kHeadDim * sizeof(float), 256));
    p.out = out;
    p.err = err;
    p.B = B;
    p.H = H;
    p.Hkv = Hkv;
    p.hpg = H / Hkv;
    p.maxC = static_cast<int>((static_cast<long long>(max_len) + kChunk - 1) / kChunk);
    p.max_len = max_len;
    p.len_add = append ? 1 : 0;
    p.pairing = rs.pairing;
    p.pages = paged ? paged->pages : nullptr;
    p.page_size = paged ? paged->page_size : 0;
    p.max_pages = paged ? paged->max_pages : 0;
    p.num_pages = paged ? paged->num_pages : 0;
    p.eps = eps;
    p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kHeadDim))) * rs.logit_mult;
    p.rf = rs.rf;

    const int h = p.hpg;
    if (h == 1) return launch_decode<1>(p, 1, st);
    if (h == 2) return launch_decode<2>(p, 1, st);
    if (h <= 4) return launch_decode<4>(p, 1, st);
    return launch_decode<8>(p, (h + 7) / 8, st);
}

}  // namespace

extern "C" gqa_status gqa_attn_decode(const void *q, const void *k_cache, const void *v_cache,
                                      const int64_t *cache_offsets, const int32_t *seqlens, const int32_t *q_pos,
                                      const float *qnorm_w, float theta, float eps, float *out, int B, int H,
                                      int Hkv, int D, int max_len, void *workspace, size_t workspace_bytes,
                                      void *stream) {
    if (!params_ok(theta, eps)) return GQA_ERR_INVALID_ARG;
    return decode_impl(q, nullptr, nullptr, const_cast<void *>(k_cache), const_cast<void *>(v_cache), cache_offsets,
                       nullptr, seqlens, q_pos, qnorm_w, nullptr, plain_rope(theta), eps, out, B, H, Hkv, D, max_len,
                       workspace, workspace_bytes, stream);
}

extern "C" gqa_status gqa_attn_decode_ex(const void *q, const void *k_cache, const void *v_cache,
                                         const int64_t *cache_offsets, const int32_t *seqlens, const int32_t *q_pos,
                                         const float *qnorm_w, const gqa_rope_config *rope, float eps, float *out,
                                         int B, int H, int Hkv, int D, int max_len, void *workspace,
                                         size_t workspace_bytes, void *stream) {
    RopeSpec rs;
    if (!rope_spec(rope, rs)) return GQA_ERR_INVALID_ARG;
    return decode_impl(q, nullptr, nullptr, const_cast<void *>(k_cache), const_cast<void *>(v_cache), cache_offsets,
                       nullptr, seqlens, q_pos, qnorm_w, nullptr, rs, eps, out, B, H, Hkv, D, max_len, workspace,
                       workspace_bytes, stream);
}

extern "C" gqa_status gqa_attn_decode_append(const void *q, const void *k_new, const void *v_new, void *k_cache,
                                             void *v_cache, const int64_t *cache_offsets, const int32_t *seqlens,
                                             const int32_t *q_pos, const float *qnorm_w, const float *knorm_w,
                                             float theta, float eps, float *out, int B, int H, int Hkv, int D,
                                             int max_len, void *workspace, size_t workspace_bytes, void *stream) {
    if (!k_new || !v_new || !knorm_w) return GQA_ERR_INVALID_ARG;
    if (!params_ok(theta, eps)) return GQA_ERR_INVALID_ARG;
    return decode_impl(q, k_new, v_new, k_cache, v_cache, cache_offsets, nullptr, seqlens, q_pos, qnorm_w, knorm_w,
                       plain_rope(theta), eps, out, B, H, Hkv, D, max_len, workspace, workspace_bytes, stream);
}

extern "C" gqa_status gqa_attn_decode_append_ex(const void *q, const void *k_new, const void *v_new, void *k_cache,
                                                void *v_cache, const int64_t *cache_offsets, const int32_t *seqlens,
                                                const int32_t *q_pos, const float *qnorm_w, const float *knorm_w,
                                                const gqa_rope_config *rope, float eps, float *out, int B, int H,
                                                int Hkv, int D, int max_len, void *workspace, size_t workspace_bytes,
                                                void *stream) {
    if (!k_new || !v_new || !knorm_w) return GQA_ERR_INVALID_ARG;
    RopeSpec rs;
    if (!rope_spec(rope, rs)) return GQA_ERR_INVALID_ARG;
    return decode_impl(q, k_new, v_new, k_cache, v_cache, cache_offsets, nullptr, seqlens, q_pos, qnorm_w, knorm_w, rs,
                       eps, out, B, H, Hkv, D, max_len, workspace, workspace_bytes, stream);
}

extern "C" gqa_status gqa_attn_decode_paged(const void *q, const void *k_pages, const void *v_pages,
                                            const int32_t *page_table, int num_pages, int page_size,
                                            int max_pages_per_seq, const int32_t *seqlens, const int32_t *q_pos,
                                            const float *qnorm_w, const gqa_rope_config *rope, float eps, float *out,
                                            int B, int H, int Hkv, int D, int max_len, void *workspace,
                                            size_t workspace_bytes, void *stream) {
    RopeSpec rs;
    if (!rope_spec(rope, rs)) return GQA_ERR_INVALID_ARG;
    const PagedCache pc{page_table, num_pages, page_size, max_pages_per_seq};
    return decode_impl(q, nullptr, nullptr, const_cast<void *>(k_pages), const_cast<void *>(v_pages), nullptr, &pc,
                       seqlens, q_pos, qnorm_w, nullptr, rs, eps, out, B, H, Hkv, D, max_len, workspace,
                       workspace_bytes, stream);
}

extern "C" gqa_status gqa_attn_decode_append_paged(const void *q, const void *k_new, const void *v_new, void *k_pages,
                                                   void *v_pages, const int32_t *page_table, int num_pages,
                                                   int page_size, int max_pages_per_seq, const int32_t *seqlens,
                                                   const int32_t *q_pos, const float *qnorm_w, const float *knorm_w,
                                                   const gqa_rope_config *rope, float eps, float *out, int B, int H,
                                                   int Hkv, int D, int max_len, void *workspace,
                                                   size_t workspace_bytes, void *stream) {
    if (!k_new || !v_new || !knorm_w) return GQA_ERR_INVALID_ARG;
    RopeSpec rs;
    if (!rope_spec(rope, rs)) return GQA_ERR_INVALID_ARG;
    const PagedCache pc{page_table, num_pages, page_size, max_pages_per_seq};
    return decode_impl(q, k_new, v_new, k_pages, v_pages, nullptr, &pc, seqlens, q_pos, qnorm_w, knorm_w, rs, eps, out,
                       B, H, Hkv, D, max_len, workspace, workspace_bytes, stream);
}

namespace {

// Scratch for gqa_attn_decode_noalloc: part of the library's own device image, so no
// call ever allocates.  Host code must not use the symbol's host-side address; the
// device address comes from cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GQA_NOALLOC_SCRATCH_BYTES];

void *noalloc_scratch_address() {
    static std::atomic<void *> cache[kMaxDevices];
    const int dev = current_device();
    if (dev < 0) return nullptr;
    void *p = cache[dev].load(std::memory_order_acquire);
    if (p) return p;
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr) return nullptr;
    cache[dev].store(addr, std::memory_order_release);
    return addr;
}

}  // namespace

extern "C" gqa_status gqa_attn_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                              const int64_t *cache_offsets, const int32_t *seqlens,
                                              const int32_t *q_pos, const float *qnorm_w, float theta, float eps,
                                              float *out, int B, int H, int Hkv, int D, int max_len,
                                              void *stream) {
    // gqa_attn_decode's argument checks first, then the size limit of the built-in
    // scratch; its device address is only looked up when there is work to launch.
    if (!params_ok(theta, eps)) return GQA_ERR_INVALID_ARG;
    bool empty = false;
    const gqa_status chk = decode_check(q, nullptr, nullptr, k_cache, v_cache, cache_offsets, nullptr, seqlens, q_pos,
                                        qnorm_w, nullptr, eps, out, B, H, Hkv, D, max_len, empty);
    if (chk != GQA_OK || empty) return chk;
    if (gqa_attn_decode_workspace_size(B, H, Hkv, D, max_len) > GQA_NOALLOC_SCRATCH_BYTES) return GQA_ERR_WORKSPACE;
    void *scratch = noalloc_scratch_address();
    if (!scratch) return GQA_ERR_CUDA;
    return gqa_attn_decode(q, k_cache, v_cache, cache_offsets, seqlens, q_pos, qnorm_w, theta, eps, out, B, H, Hkv,
                           D, max_len, scratch, GQA_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" void gqa_attn_test_stall(int enable) { g_test_stall.store(enable ? 1 : 0, std::memory_order_relaxed); }

extern "C" gqa_status gqa_attn_device_status(void *stream) {
    unsigned *err = device_error_word();
    if (!err) return GQA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned h = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess) return GQA_ERR_CUDA;
    if (cudaMemcpyAsync(&h, err, sizeof h, cudaMemcpyDeviceToHost, st) != cudaSuccess) return GQA_ERR_CUDA;
    if (cudaMemsetAsync(err, 0, sizeof h, st) != cudaSuccess) return GQA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return GQA_ERR_CUDA;
    if (h & kErrTimeout) return GQA_ERR_DEVICE_TIMEOUT;
    if (h & kErrInput) return GQA_ERR_DEVICE_INPUT;
    return GQA_OK;
}
