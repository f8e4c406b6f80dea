// libkvq C ABI: argument validation, launch selection, workspace sizing and
// the status word.  No allocation happens here or in any kernel; the only
// state kept is a per-device cache of the SM count.
#include <atomic>
#include <limits.h>

#include "kvq_internal.cuh"


using namespace kvq;

namespace {

constexpr int SPLIT_CTAS_PER_SM = 1;     // one split CTA (four groups) per SM
constexpr int MIN_BLOCKS_PER_CTA = 64;   // 1024 tokens: below this, fewer CTAs

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

int device_sm_count() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < 64) {
        const int c = cached[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

kvq_status check_cache(const kvq_cache_desc *c) {
    if (!c) return KVQ_ERR_INVALID_ARG;
    if (c->head_dim != D || c->group != GS) return KVQ_ERR_UNSUPPORTED;
    if (c->B < 1 || c->Hkv < 1 || c->capacity < BLK_TOK || c->capacity % BLK_TOK != 0)
        return KVQ_ERR_INVALID_ARG;
    if (c->sink_fp16 < 0 || c->sink_fp16 > MAX_SINK || c->sink_fp16 > c->capacity)
        return KVQ_ERR_INVALID_ARG;
    if (!c->blocks || !c->status) return KVQ_ERR_INVALID_ARG;
    if (!aligned(c->blocks, 16) || !aligned(c->status, 8)) return KVQ_ERR_UNSUPPORTED;
    if (c->sink_fp16 > 0) {
        if (!c->k_sink || !c->v_sink) return KVQ_ERR_INVALID_ARG;
        if (!aligned(c->k_sink, 16) || !aligned(c->v_sink, 16)) return KVQ_ERR_UNSUPPORTED;
    }
    if ((long long)c->B * c->Hkv * (c->capacity / BLK_TOK) > INT_MAX) return KVQ_ERR_INVALID_ARG;
    if (c->B > 32767) return KVQ_ERR_INVALID_ARG;
    if (c->block_table) {
        if (!aligned(c->block_table, 4)) return KVQ_ERR_UNSUPPORTED;
        if (c->num_blocks < 1 || (long long)c->num_blocks * c->Hkv > INT_MAX) return KVQ_ERR_INVALID_ARG;
    }
    if (c->sink_pos) {                       // identified sinks
        if (c->sink_fp16 < 1 || !c->sink_count) return KVQ_ERR_INVALID_ARG;
        if (!aligned(c->sink_pos, 4) || !aligned(c->sink_count, 4)) return KVQ_ERR_UNSUPPORTED;
    }
    return KVQ_OK;
}

kvq_status check_rot(kvq_rot_mode mode, const float *R_k, const float *R_v, const int32_t *perm) {
    if (mode == KVQ_ROT_DENSE) {
        if (!R_k || !R_v) return KVQ_ERR_INVALID_ARG;
        if (!aligned(R_k, 16) || !aligned(R_v, 16)) return KVQ_ERR_UNSUPPORTED;
    } else if (mode == KVQ_ROT_PERM_FWHT) {
        if (!perm) return KVQ_ERR_INVALID_ARG;
        if (!aligned(perm, 16)) return KVQ_ERR_UNSUPPORTED;
    } else {
        return KVQ_ERR_INVALID_ARG;
    }
    return KVQ_OK;
}

int split_ctas(int B, int Hkv, int max_ctx, int sms) {
    const long long blocks = (long long)B * Hkv * ((max_ctx + BLK_TOK - 1) / BLK_TOK);
    long long want = (blocks + MIN_BLOCKS_PER_CTA - 1) / MIN_BLOCKS_PER_CTA;
    const long long cap = (long long)sms * SPLIT_CTAS_PER_SM;
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    return (int)want;
}

}  // namespace

extern "C" {

size_t kvq_cache_bytes(int32_t B, int32_t Hkv, int32_t capacity) {
    if (B < 1 || Hkv < 1 || capacity < BLK_TOK || capacity % BLK_TOK) return 0;
    return (size_t)B * Hkv * (capacity / BLK_TOK) * BLK_BYTES;
}

}  // extern "C"

namespace {

// Argument checks of an append (nothing is launched).
kvq_status append_check(const uint16_t *K, const uint16_t *V, int32_t T, kvq_rot_mode mode,
                        const float *R_k, const float *R_v, const int32_t *perm,
                        const kvq_cache_desc *cache, const int32_t *seq_lens) {
    kvq_status s = check_cache(cache);
    if (s != KVQ_OK) return s;
    if ((s = check_rot(mode, R_k, R_v, perm)) != KVQ_OK) return s;
    if (T < 0 || !seq_lens || !aligned(seq_lens, 4)) return KVQ_ERR_INVALID_ARG;
    if (T == 0) return KVQ_OK;
    if (!K || !V) return KVQ_ERR_INVALID_ARG;
    if (!aligned(K, 16) || !aligned(V, 16)) return KVQ_ERR_UNSUPPORTED;
    if (T > cache->capacity) return KVQ_ERR_INVALID_ARG;
    return KVQ_OK;
}

// The append's kernel, arguments already checked.
kvq_status append_launch(const uint16_t *K, const uint16_t *V, int32_t T, kvq_rot_mode mode,
                         const float *R_k, const float *R_v, const int32_t *perm,
                         const kvq_cache_desc *cache, int32_t *seq_lens, void *stream) {
    if (T == 0) return KVQ_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = append_tc_eligible(mode, K, V, T, cache->B)
                        ? launch_append_tc(K, V, T, mode, R_k, R_v, perm, *cache, seq_lens, st)
                        : launch_append_small(K, V, T, mode, R_k, R_v, perm, *cache, seq_lens, st);
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace

extern "C" {

kvq_status kvq_rotate_quantize_append(const uint16_t *K, const uint16_t *V, int32_t T,
                                      kvq_rot_mode mode, const float *R_k, const float *R_v,
                                      const int32_t *perm, const kvq_cache_desc *cache,
                                      int32_t *seq_lens, void *stream) {
    const kvq_status s = append_check(K, V, T, mode, R_k, R_v, perm, cache, seq_lens);
    if (s != KVQ_OK) return s;
    return append_launch(K, V, T, mode, R_k, R_v, perm, cache, seq_lens, stream);
}

kvq_status kvq_identify_sinks(const float *act, int32_t T, float tau, const kvq_cache_desc *cache,
                              const int32_t *seq_lens, void *stream) {
    kvq_status s = check_cache(cache);
    if (s != KVQ_OK) return s;
    if (!cache->sink_pos || !act || !seq_lens || T < 1) return KVQ_ERR_INVALID_ARG;
    if (!aligned(act, 4) || !aligned(seq_lens, 4)) return KVQ_ERR_UNSUPPORTED;
    if (T > cache->capacity) return KVQ_ERR_INVALID_ARG;
    const cudaError_t e =
        launch_identify_sinks(act, T, tau, *cache, seq_lens, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

static bool gh_ok(int gh, int Hkv) {
    return (gh == 1 || gh == 2 || gh == 4 || gh == 8) && Hkv % gh == 0;
}

kvq_status kvq_prerope_append(const uint16_t *K, const uint16_t *V, int32_t T, int32_t group_heads,
                              const int32_t *perm, const kvq_cache_desc *cache, int32_t *seq_lens,
                              void *stream) {
    kvq_status s = check_cache(cache);
    if (s != KVQ_OK) return s;
    if (!gh_ok(group_heads, cache->Hkv)) return KVQ_ERR_UNSUPPORTED;
    if (!perm || T < 0 || !seq_lens || !aligned(seq_lens, 4)) return KVQ_ERR_INVALID_ARG;
    if (!aligned(perm, 16)) return KVQ_ERR_UNSUPPORTED;
    if (T == 0) return KVQ_OK;
    if (!K || !V) return KVQ_ERR_INVALID_ARG;
    if (!aligned(K, 16) || !aligned(V, 16)) return KVQ_ERR_UNSUPPORTED;
    if (T > cache->capacity) return KVQ_ERR_INVALID_ARG;
    const cudaError_t e = launch_append_prerope(K, V, T, group_heads, perm, *cache, seq_lens,
                                                static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

size_t kvq_prerope_workspace_size(int32_t B, int32_t Hq, int32_t Hkv, int32_t group_heads,
                                  int32_t max_ctx, int32_t sm_count) {
    if (B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv || max_ctx < 1 || sm_count < 1) return 0;
    if (!gh_ok(group_heads, Hkv)) return 0;
    return prerope_ws_bytes(B, Hq, Hkv, group_heads, max_ctx, sm_count);
}

kvq_status kvq_prerope_decode(const uint16_t *Q, int32_t Hq, const kvq_cache_desc *cache,
                              int32_t group_heads, const int32_t *perm, float rope_base,
                              const int32_t *seq_lens, int32_t max_ctx, void *workspace,
                              size_t ws_bytes, uint16_t *out, void *stream) {
    kvq_status s = check_cache(cache);
    if (s != KVQ_OK) return s;
    if (!gh_ok(group_heads, cache->Hkv)) return KVQ_ERR_UNSUPPORTED;
    if (!Q || !out || !seq_lens || !workspace || !perm) return KVQ_ERR_INVALID_ARG;
    if (!aligned(Q, 16) || !aligned(out, 16) || !aligned(workspace, 256) ||
        !aligned(seq_lens, 4) || !aligned(perm, 16))
        return KVQ_ERR_UNSUPPORTED;
    if (Hq < cache->Hkv || Hq % cache->Hkv != 0 || Hq > 65535) return KVQ_ERR_INVALID_ARG;
    const int G = Hq / cache->Hkv;
    if ((G != 1 && G != 2 && G != 4 && G != 8) || G * group_heads > 8) return KVQ_ERR_UNSUPPORTED;
    if (!(rope_base > 1.0f) || !(rope_base < 3.0e38f)) return KVQ_ERR_INVALID_ARG;
    if (max_ctx < 1 || max_ctx > cache->capacity) return KVQ_ERR_INVALID_ARG;
    const int sms = device_sm_count();
    if (sms < 1) return KVQ_ERR_CUDA;
    if (ws_bytes < prerope_ws_bytes(cache->B, Hq, cache->Hkv, group_heads, max_ctx, sms))
        return KVQ_ERR_WORKSPACE;
    const cudaError_t e = launch_decode_prerope(Q, Hq, *cache, group_heads, perm, rope_base,
                                                seq_lens, max_ctx, sms, workspace, out,
                                                static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_debug_rotate_group_f32(const uint16_t *X, int32_t N, int32_t group_heads,
                                      const int32_t *perm, float *Xrot, void *stream) {
    if (!X || !Xrot || !perm || N < 0) return KVQ_ERR_INVALID_ARG;
    if (group_heads != 1 && group_heads != 2 && group_heads != 4 && group_heads != 8)
        return KVQ_ERR_UNSUPPORTED;
    if (!aligned(X, 16) || !aligned(Xrot, 16) || !aligned(perm, 16)) return KVQ_ERR_UNSUPPORTED;
    if (N == 0) return KVQ_OK;
    const cudaError_t e = launch_debug_rotate_group(X, N, group_heads, perm, Xrot,
                                                    static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

size_t kvq_decode_workspace_size(int32_t B, int32_t Hq, int32_t Hkv, int32_t max_ctx,
                                 int32_t sm_count) {
    if (B < 1 || Hkv < 1 || Hq < Hkv || Hq % Hkv || max_ctx < 1 || sm_count < 1) return 0;
    const int C = split_ctas(B, Hkv, max_ctx, sm_count);
    return ws_layout(B, Hq, Hkv, C).total;
}

}  // extern "C"

namespace {

// Argument checks of a decode (nothing is launched); C = split CTAs.
kvq_status decode_check(const uint16_t *Q, int32_t Hq, int32_t q_len, uint32_t flags,
                        const kvq_cache_desc *cache, kvq_rot_mode mode, const float *R_k,
                        const float *R_v, const int32_t *perm, const int32_t *seq_lens,
                        int32_t sink_fp16, int32_t max_ctx, const void *workspace,
                        size_t ws_bytes, const uint16_t *out, int &C) {
    kvq_status s = check_cache(cache);
    if (s != KVQ_OK) return s;
    if ((s = check_rot(mode, R_k, R_v, perm)) != KVQ_OK) return s;
    if (!Q || !out || !seq_lens || !workspace) return KVQ_ERR_INVALID_ARG;
    if (!aligned(Q, 16) || !aligned(out, 16) || !aligned(workspace, 256) || !aligned(seq_lens, 4))
        return KVQ_ERR_UNSUPPORTED;
    if (q_len < 1 || q_len > 8 || (flags & ~KVQ_DECODE_OUT_ROTATED) != 0) return KVQ_ERR_INVALID_ARG;
    if (Hq < cache->Hkv || Hq % cache->Hkv != 0 || (long long)Hq * q_len > 65535)
        return KVQ_ERR_INVALID_ARG;
    const int Hqq = Hq * q_len;                     // query rows per sequence
    const int G = Hqq / cache->Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return KVQ_ERR_UNSUPPORTED;
    if (sink_fp16 != cache->sink_fp16) return KVQ_ERR_INVALID_ARG;
    if (max_ctx < q_len || max_ctx > cache->capacity) return KVQ_ERR_INVALID_ARG;
    const int sms = device_sm_count();
    if (sms < 1) return KVQ_ERR_CUDA;
    C = split_ctas(cache->B, cache->Hkv, max_ctx, sms);
    if (ws_bytes < ws_layout(cache->B, Hqq, cache->Hkv, C).total) return KVQ_ERR_WORKSPACE;
    return KVQ_OK;
}

// Shared body of the decode entry points: q_len queries per sequence (Hq
// heads each), options in flags, optional events around the split kernel.
kvq_status decode_impl(const uint16_t *Q, int32_t Hq, int32_t q_len, uint32_t flags,
                       const kvq_cache_desc *cache, kvq_rot_mode mode, const float *R_k,
                       const float *R_v, const int32_t *perm, const int32_t *seq_lens,
                       int32_t sink_fp16, int32_t max_ctx, void *workspace, size_t ws_bytes,
                       uint16_t *out, void *stream, void *ev_begin, void *ev_end,
                       const KeyAdapter &ad = KeyAdapter()) {
    int C = 0;
    const kvq_status s = decode_check(Q, Hq, q_len, flags, cache, mode, R_k, R_v, perm, seq_lens,
                                      sink_fp16, max_ctx, workspace, ws_bytes, out, C);
    if (s != KVQ_OK) return s;
    cudaError_t e = launch_decode(Q, Hq * q_len, *cache, mode, R_k, R_v, perm, seq_lens, C,
                                  workspace, out, static_cast<cudaStream_t>(stream),
                                  static_cast<cudaEvent_t>(ev_begin), static_cast<cudaEvent_t>(ev_end),
                                  q_len, (flags & KVQ_DECODE_OUT_ROTATED) ? 1 : 0, ad);
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // namespace

extern "C" {

kvq_status kvq_decode_attention_timed(const uint16_t *Q, int32_t Hq, const kvq_cache_desc *cache,
                                      kvq_rot_mode mode, const float *R_k, const float *R_v,
                                      const int32_t *perm, const int32_t *seq_lens,
                                      int32_t sink_fp16, int32_t max_ctx, void *workspace,
                                      size_t ws_bytes, uint16_t *out, void *stream, void *ev_begin,
                                      void *ev_end) {
    return decode_impl(Q, Hq, 1, 0u, cache, mode, R_k, R_v, perm, seq_lens, sink_fp16, max_ctx,
                       workspace, ws_bytes, out, stream, ev_begin, ev_end);
}

kvq_status kvq_decode_attention_ex(const uint16_t *Q, int32_t Hq, int32_t q_len, uint32_t flags,
                                   const kvq_cache_desc *cache, kvq_rot_mode mode, const float *R_k,
                                   const float *R_v, const int32_t *perm, const int32_t *seq_lens,
                                   int32_t sink_fp16, int32_t max_ctx, void *workspace,
                                   size_t ws_bytes, uint16_t *out, void *stream) {
    return decode_impl(Q, Hq, q_len, flags, cache, mode, R_k, R_v, perm, seq_lens, sink_fp16,
                       max_ctx, workspace, ws_bytes, out, stream, nullptr, nullptr);
}

kvq_status kvq_decode_attention_adapter(const uint16_t *Q, int32_t Hq, int32_t q_len,
                                        uint32_t flags, const kvq_cache_desc *cache,
                                        kvq_rot_mode mode, const float *R_k, const float *R_v,
                                        const int32_t *perm, const float *U_k, const float *V_k,
                                        int32_t rank, const int32_t *seq_lens, int32_t sink_fp16,
                                        int32_t max_ctx, void *workspace, size_t ws_bytes,
                                        uint16_t *out, void *stream) {
    if (!U_k || !V_k || rank < 1 || rank > 128) return KVQ_ERR_INVALID_ARG;
    if (!aligned(U_k, 4) || !aligned(V_k, 4)) return KVQ_ERR_UNSUPPORTED;
    KeyAdapter ad;
    ad.U = U_k;
    ad.V = V_k;
    ad.r = rank;
    return decode_impl(Q, Hq, q_len, flags, cache, mode, R_k, R_v, perm, seq_lens, sink_fp16,
                       max_ctx, workspace, ws_bytes, out, stream, nullptr, nullptr, ad);
}

kvq_status kvq_append_decode(const uint16_t *K, const uint16_t *V, int32_t T, const uint16_t *Q,
                             int32_t Hq, const kvq_cache_desc *cache, kvq_rot_mode mode,
                             const float *R_k, const float *R_v, const int32_t *perm,
                             int32_t *seq_lens, int32_t max_ctx, void *workspace, size_t ws_bytes,
                             uint16_t *out, void *stream) {
    kvq_status s = append_check(K, V, T, mode, R_k, R_v, perm, cache, seq_lens);
    if (s != KVQ_OK) return s;
    int C = 0;
    s = decode_check(Q, Hq, 1, 0u, cache, mode, R_k, R_v, perm, seq_lens, cache->sink_fp16,
                     max_ctx, workspace, ws_bytes, out, C);
    if (s != KVQ_OK) return s;
    if ((s = append_launch(K, V, T, mode, R_k, R_v, perm, cache, seq_lens, stream)) != KVQ_OK)
        return s;
    const cudaError_t e = launch_decode(Q, Hq, *cache, mode, R_k, R_v, perm, seq_lens, C, workspace,
                                        out, static_cast<cudaStream_t>(stream), nullptr, nullptr, 1, 0);
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // extern "C"

namespace {

// Staging layout of the host-buffer step, after the decode workspace:
// K, V [B][T][Hkv][128], Q and out [B][Hq][128], each 256-B aligned.
struct StepLayout {
    size_t k, v, q, out, total;
};
StepLayout step_layout(int B, int T, int Hq, int Hkv, size_t dec_ws) {
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    StepLayout l;
    const size_t kv = (size_t)B * T * Hkv * D * 2, qb = (size_t)B * Hq * D * 2;
    l.k = up(dec_ws);
    l.v = up(l.k + kv);
    l.q = up(l.v + kv);
    l.out = up(l.q + qb);
    l.total = up(l.out + qb);
    return l;
}

}  // namespace

extern "C" {

size_t kvq_step_workspace_size(int32_t B, int32_t T, int32_t Hq, int32_t Hkv, int32_t max_ctx,
                               int32_t sm_count) {
    if (T < 1) return 0;
    const size_t dec = kvq_decode_workspace_size(B, Hq, Hkv, max_ctx, sm_count);
    if (dec == 0) return 0;
    return step_layout(B, T, Hq, Hkv, dec).total;
}

kvq_status kvq_append_decode_host(const uint16_t *K_host, const uint16_t *V_host, int32_t T,
                                  const uint16_t *Q_host, int32_t Hq, const kvq_cache_desc *cache,
                                  kvq_rot_mode mode, const float *R_k, const float *R_v,
                                  const int32_t *perm, int32_t *seq_lens, int32_t max_ctx,
                                  void *workspace, size_t ws_bytes, uint16_t *out_host,
                                  void *stream) {
    kvq_status s = check_cache(cache);
    if (s != KVQ_OK) return s;
    if (!K_host || !V_host || !Q_host || !out_host || !workspace || T < 1) return KVQ_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return KVQ_ERR_UNSUPPORTED;
    if (Hq < cache->Hkv || Hq % cache->Hkv != 0) return KVQ_ERR_INVALID_ARG;
    const int sms = device_sm_count();
    if (sms < 1) return KVQ_ERR_CUDA;
    const size_t dec = kvq_decode_workspace_size(cache->B, Hq, cache->Hkv, max_ctx, sms);
    if (dec == 0) return KVQ_ERR_INVALID_ARG;
    const StepLayout l = step_layout(cache->B, T, Hq, cache->Hkv, dec);
    if (ws_bytes < l.total) return KVQ_ERR_WORKSPACE;
    uint8_t *w = static_cast<uint8_t *>(workspace);
    uint16_t *K = reinterpret_cast<uint16_t *>(w + l.k), *V = reinterpret_cast<uint16_t *>(w + l.v);
    uint16_t *Q = reinterpret_cast<uint16_t *>(w + l.q), *out = reinterpret_cast<uint16_t *>(w + l.out);
    // every check of the two device calls before the first copy
    if ((s = append_check(K, V, T, mode, R_k, R_v, perm, cache, seq_lens)) != KVQ_OK) return s;
    int C = 0;
    if ((s = decode_check(Q, Hq, 1, 0u, cache, mode, R_k, R_v, perm, seq_lens, cache->sink_fp16,
                          max_ctx, workspace, dec, out, C)) != KVQ_OK)
        return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t kv = (size_t)cache->B * T * cache->Hkv * D * 2, qb = (size_t)cache->B * Hq * D * 2;
    // kv and qb are multiples of 256 B, so the K, V and Q regions of the
    // workspace are back to back: host inputs that are back to back as well
    // (views of one pinned buffer) go in with a single copy
    const uint8_t *hk = reinterpret_cast<const uint8_t *>(K_host);
    const bool one = reinterpret_cast<const uint8_t *>(V_host) == hk + kv &&
                     reinterpret_cast<const uint8_t *>(Q_host) == hk + 2 * kv && l.v == l.k + kv &&
                     l.q == l.v + kv;
    // Adjacent host inputs may still be separate allocations (a caching host
    // allocator can place them back to back): if the single copy is refused,
    // the three copies are made instead.
    bool copied = false;
    if (one) {
        copied = cudaMemcpyAsync(K, K_host, 2 * kv + qb, cudaMemcpyHostToDevice, st) == cudaSuccess;
        if (!copied) (void)cudaGetLastError();
    }
    if (!copied && (cudaMemcpyAsync(K, K_host, kv, cudaMemcpyHostToDevice, st) != cudaSuccess ||
                    cudaMemcpyAsync(V, V_host, kv, cudaMemcpyHostToDevice, st) != cudaSuccess ||
                    cudaMemcpyAsync(Q, Q_host, qb, cudaMemcpyHostToDevice, st) != cudaSuccess)) {
        return KVQ_ERR_CUDA;
    }
    if ((s = append_launch(K, V, T, mode, R_k, R_v, perm, cache, seq_lens, stream)) != KVQ_OK) return s;
    if (launch_decode(Q, Hq, *cache, mode, R_k, R_v, perm, seq_lens, C, workspace, out, st, nullptr,
                      nullptr, 1, 0) != cudaSuccess)
        return KVQ_ERR_CUDA;
    return cudaMemcpyAsync(out_host, out, qb, cudaMemcpyDeviceToHost, st) == cudaSuccess ? KVQ_OK
                                                                                      : KVQ_ERR_CUDA;
}

kvq_status kvq_decode_attention(const uint16_t *Q, int32_t Hq, const kvq_cache_desc *cache,
                                kvq_rot_mode mode, const float *R_k, const float *R_v,
                                const int32_t *perm, const int32_t *seq_lens,
                                int32_t sink_fp16, int32_t max_ctx, void *workspace,
                                size_t ws_bytes, uint16_t *out, void *stream) {
    return kvq_decode_attention_timed(Q, Hq, cache, mode, R_k, R_v, perm, seq_lens, sink_fp16,
                                      max_ctx, workspace, ws_bytes, out, stream, nullptr, nullptr);
}

kvq_status kvq_get_status(const kvq_cache_desc *cache, void *stream, int32_t *host_out) {
    if (!cache || !cache->status || !host_out) return KVQ_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(host_out, cache->status, sizeof(int32_t), cudaMemcpyDeviceToHost, st) !=
        cudaSuccess)
        return KVQ_ERR_CUDA;
    return cudaStreamSynchronize(st) == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_clear_status(const kvq_cache_desc *cache, void *stream) {
    if (!cache || !cache->status) return KVQ_ERR_INVALID_ARG;
    return cudaMemsetAsync(cache->status, 0, 2 * sizeof(int32_t), static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? KVQ_OK
               : KVQ_ERR_CUDA;
}

kvq_status kvq_debug_rotate_f32(const uint16_t *X, int32_t N, kvq_rot_mode mode, const float *R,
                                const int32_t *perm, int32_t variant, float *Xrot, void *stream) {
    if (!X || !Xrot || N < 0) return KVQ_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(Xrot, 16)) return KVQ_ERR_UNSUPPORTED;
    kvq_status s = check_rot(mode, R, R, perm);
    if (s != KVQ_OK) return s;
    if (variant != 0 && variant != 1) return KVQ_ERR_INVALID_ARG;
    if (N == 0) return KVQ_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = variant == 1
                        ? launch_debug_rotate_tc(X, N, mode, R, perm, Xrot, st)
                        : launch_debug_rotate_small(X, N, mode, R, perm, Xrot, st);
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_debug_quantize_f32(const float *Xrot, int32_t N, uint8_t *codes, uint16_t *meta,
                                  void *stream) {
    if (!Xrot || !codes || !meta || N < 0) return KVQ_ERR_INVALID_ARG;
    if (!aligned(Xrot, 16) || !aligned(codes, 4) || !aligned(meta, 4)) return KVQ_ERR_UNSUPPORTED;
    if (N == 0) return KVQ_OK;
    cudaError_t e = launch_debug_quantize(Xrot, N, codes, meta, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_debug_wait_timeout(const void *src, uint32_t poll_limit, int32_t *status,
                                  int32_t *result, void *stream) {
    if (!src || !status || !result || poll_limit == 0) return KVQ_ERR_INVALID_ARG;
    if (!aligned(src, 16) || !aligned(status, 4) || !aligned(result, 4)) return KVQ_ERR_UNSUPPORTED;
    cudaError_t e = launch_debug_wait_timeout(static_cast<const uint8_t *>(src), poll_limit, status,
                                              result, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

const char *kvq_status_string(kvq_status s) {
    switch (s) {
        case KVQ_OK: return "ok";
        case KVQ_ERR_INVALID_ARG: return "invalid argument";
        case KVQ_ERR_UNSUPPORTED: return "unsupported shape or alignment";
        case KVQ_ERR_CUDA: return "CUDA error";
        case KVQ_ERR_CAPACITY: return "capacity exceeded";
        case KVQ_ERR_WORKSPACE: return "workspace too small";
    }
    return "unknown status";
}

}  // extern "C"
