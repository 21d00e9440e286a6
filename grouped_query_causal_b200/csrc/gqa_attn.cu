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

#include "gqa_attn.h"
#include "decode.cuh"
#include "prefill.cuh"

namespace gqa {

// The device status word: error bits set by kernels (kErrTimeout, kErrInput).
__device__ unsigned g_device_error = 0;

namespace {

constexpr int kMaxDevices = 64;

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

// 4-D bf16 tensor [d3][d2][d1][d0] (d0 innermost, contiguous), box (64, 1, 128, 1),
// 128-byte swizzle, zero fill outside the tensor.
bool make_bf16_map(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {d0, d1, d2, d3};
    const cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
    const cuuint32_t box[4] = {64, 1, 128, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
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
    if (cudaFuncSetAttribute(attn_fwd_kernel<kPairAdjacent>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess ||
        cudaFuncSetAttribute(attn_fwd_kernel<kPairHalf>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess)
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

// Enqueue the k-hat prologue (arguments already validated).
gqa_status launch_k_norm_rope(const void *k, const int32_t *pos, const float *knorm_w, const RopeSpec &rs,
                              float eps, void *k_hat, float *rope_cs, long long ntok, int Hkv, cudaStream_t st) {
    KPrologueParams kp;
    kp.k = static_cast<const uint16_t *>(k);
    kp.pos = pos;
    kp.wk = knorm_w;
    kp.khat = static_cast<uint16_t *>(k_hat);
    kp.rope_cs = rope_cs;
    kp.ntok = ntok;
    kp.Hkv = Hkv;
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

// Enqueue the attention kernel (arguments already validated).
gqa_status launch_attention(const void *q, const void *k_hat, const void *v, const int32_t *pos,
                            const float *rope_cs, const float *qnorm_w, const RopeSpec &rs, float eps, float *out,
                            int B, int T, int H, int Hkv, cudaStream_t st) {
    unsigned *err = device_error_word();
    if (!err) return GQA_ERR_CUDA;
    CUtensorMap tm_q, tm_k, tm_v;
    if (!make_bf16_map(&tm_q, q, kHeadDim, H, T, B) || !make_bf16_map(&tm_k, k_hat, kHeadDim, Hkv, T, B) ||
        !make_bf16_map(&tm_v, v, kHeadDim, Hkv, T, B))
        return GQA_ERR_CUDA;
    if (!attn_smem_attr_set()) return GQA_ERR_CUDA;
    AttnParams ap;
    ap.pos = pos;
    ap.rope_cs = rope_cs;
    ap.wq = qnorm_w;
    ap.out = out;
    ap.err = err;
    ap.B = B;
    ap.T = T;
    ap.H = H;
    ap.Hkv = Hkv;
    ap.hpg = H / Hkv;
    ap.nqb = (T + kBM - 1) / kBM;
    ap.npairs = (ap.hpg + 1) / 2;
    ap.eps = eps;
    ap.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kHeadDim))) * rs.logit_mult;
    ap.rf = rs.rf;
    const long long jobs = static_cast<long long>(ap.nqb) * B * Hkv * ap.npairs;
    if (jobs <= 0 || jobs > 0x7fffffffLL) return GQA_ERR_INVALID_ARG;
    if (rs.pairing == kPairHalf)
        attn_fwd_kernel<kPairHalf><<<static_cast<unsigned>(jobs), kAttnThreads, kSmemBytes, st>>>(tm_q, tm_k, tm_v, ap);
    else
        attn_fwd_kernel<kPairAdjacent><<<static_cast<unsigned>(jobs), kAttnThreads, kSmemBytes, st>>>(tm_q, tm_k, tm_v,
                                                                                                   ap);
    return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
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
    return launch_k_norm_rope(k, pos, knorm_w, rs, eps, k_hat, rope_cs, N, Hkv, static_cast<cudaStream_t>(stream));
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
    return launch_attention(q, k_hat, v, pos, rope_cs, qnorm_w, rs, eps, out, B, T, H, Hkv,
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
    gqa_status s =
        launch_k_norm_rope(k, pos, knorm_w, rs, eps, workspace, table, static_cast<long long>(B) * T, Hkv, st);
    if (s != GQA_OK) return s;
    return launch_attention(q, workspace, v, pos, table, qnorm_w, rs, eps, out, B, T, H, Hkv, st);
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

gqa_status decode_impl(const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                       const int64_t *cache_offsets, const PagedCache *paged, const int32_t *seqlens,
                       const int32_t *q_pos,
                       const float *qnorm_w, const float *knorm_w, const RopeSpec &rs, float eps, float *out, int B,
                       int H, int Hkv, int D, int max_len, void *workspace, size_t workspace_bytes, void *stream) {
    const bool append = k_new != nullptr || v_new != nullptr || knorm_w != nullptr;
    if (D != kHeadDim) return D > 0 ? GQA_ERR_UNSUPPORTED : GQA_ERR_INVALID_ARG;
    if (B < 0 || H <= 0 || Hkv <= 0 || H % Hkv != 0) return GQA_ERR_INVALID_ARG;
    if (!eps_ok(eps)) return GQA_ERR_INVALID_ARG;
    if (B == 0) return GQA_OK;
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
    if (D == kHeadDim && B > 0 && H > 0 && Hkv > 0 && H % Hkv == 0 && max_len > 0 &&
        gqa_attn_decode_workspace_size(B, H, Hkv, D, max_len) > GQA_NOALLOC_SCRATCH_BYTES)
        return GQA_ERR_WORKSPACE;
    // Every other argument check is gqa_attn_decode's; the scratch address is only
    // looked up when there is work to launch.
    if (D != kHeadDim || B <= 0 || H <= 0 || Hkv <= 0 || H % Hkv != 0 || max_len <= 0)
        return gqa_attn_decode(q, k_cache, v_cache, cache_offsets, seqlens, q_pos, qnorm_w, theta, eps, out, B, H,
                               Hkv, D, max_len, nullptr, 0, stream);
    void *scratch = noalloc_scratch_address();
    if (!scratch) return GQA_ERR_CUDA;
    return gqa_attn_decode(q, k_cache, v_cache, cache_offsets, seqlens, q_pos, qnorm_w, theta, eps, out, B, H, Hkv,
                           D, max_len, scratch, GQA_NOALLOC_SCRATCH_BYTES, stream);
}

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
