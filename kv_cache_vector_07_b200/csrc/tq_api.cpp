// C-ABI entry points of libtqkv: argument validation, workspace sizing and
// dispatch to the kernel launchers.  See include/tqkv.h for the contract.
#include <cstring>

#include <cuda_runtime.h>

#include "tq_internal.h"

namespace {

bool valid_desc(const tq_cache_desc *c) {
    if (!c) return false;
    const int d = c->d;
    if (d < 8 || d > 1024 || (d & (d - 1))) return false;
    auto half_ok = [&](int b) { return (b & ~TQ_BITS_HALF) >= 1 && (b & ~TQ_BITS_HALF) <= 3 && d >= 16 && d <= 256; };
    const bool kh = (c->kbits & TQ_BITS_HALF) != 0, vh = (c->vbits & TQ_BITS_HALF) != 0;
    const bool polar_ok = d >= 8 && d <= 256;
    if (c->kbits == TQ_BITS_POLAR ? !polar_ok
        : (kh ? !half_ok(c->kbits) : !(c->kbits == 1 || c->kbits == 2 || c->kbits == 3 || c->kbits == 4 ||
                                       c->kbits == 8)))
        return false;
    if (c->kqjl != 0 && c->kqjl != 1) return false;
    if (c->kbits == 8 && c->kqjl) return false;
    if (c->vbits == TQ_BITS_POLAR ? !polar_ok : (vh ? !half_ok(c->vbits) : (c->vbits < 0 || c->vbits > 4)))
        return false;
    if (c->page_tokens < 8 || c->page_tokens > 256 || (c->page_tokens % 8)) return false;
    if (c->n_kv_heads < 1) return false;
    return true;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int cuda_status(int e) { return e == cudaSuccess ? TQ_OK : TQ_ECUDA; }

}  // namespace

extern "C" int tq_cache_bytes(const tq_cache_desc *desc, size_t *page_bytes) {
    if (!valid_desc(desc) || !page_bytes) return TQ_EINVAL;
    tq::Layout L;
    tq::make_layout(*desc, &L);
    *page_bytes = size_t(L.page_bytes);
    return TQ_OK;
}

extern "C" size_t tq_encode_workspace_bytes(const tq_cache_desc *desc, int64_t n_tokens) {
    if (!valid_desc(desc) || n_tokens < 0) return 0;
    tq::Layout L;
    tq::make_layout(*desc, &L);
    return tq::encode_ws_bytes(L, n_tokens);
}

extern "C" int tq_encode(const tq_params *kp, const tq_params *vp, const tq_cache_desc *desc, const void *K,
                         const void *V, int in_dtype, int64_t n_tokens, const int32_t *slot_mapping, void *cache,
                         int64_t num_blocks, void *workspace, size_t workspace_bytes, void *stream) {
    if (!valid_desc(desc) || !kp || n_tokens < 0 || num_blocks < 0) return TQ_EINVAL;
    if (in_dtype != TQ_DTYPE_BF16 && in_dtype != TQ_DTYPE_F32) return TQ_EINVAL;
    if (kp->d != desc->d || kp->bits != desc->kbits) return TQ_EINVAL;
    if (desc->vbits > 0 && (!vp || vp->d != desc->d || vp->bits != desc->vbits || !V)) return TQ_EINVAL;
    if (!K || !slot_mapping || !cache || !workspace) return TQ_EINVAL;
    if (!aligned(K, 16) || (V && !aligned(V, 16)) || !aligned(cache, 256) || !aligned(workspace, 256))
        return TQ_EINVAL;
    tq::Layout L;
    tq::make_layout(*desc, &L);
    if (workspace_bytes < tq::encode_ws_bytes(L, n_tokens)) return TQ_EINVAL;
    if (n_tokens == 0) return TQ_OK;
    return cuda_status(tq::launch_encode(kp, desc->vbits > 0 ? vp : nullptr, L, K, V, in_dtype, n_tokens,
                                         slot_mapping, static_cast<uint8_t *>(cache), num_blocks,
                                         static_cast<uint8_t *>(workspace), workspace_bytes, stream));
}

namespace {

bool attn_params_ok(const tq_params *kp, const tq_params *vp, const tq_cache_desc *desc, int Hq) {
    if (!valid_desc(desc) || !kp || !vp) return false;
    if (desc->d > 256) return false;
    if (desc->vbits == 0) return false;
    if (kp->d != desc->d || kp->bits != desc->kbits || vp->d != desc->d || vp->bits != desc->vbits) return false;
    if (Hq < 1 || Hq % desc->n_kv_heads) return false;
    const int G = Hq / desc->n_kv_heads;
    if (G > 8) return false;
    return true;
}

}  // namespace

extern "C" size_t tq_decode_workspace_bytes(const tq_cache_desc *desc, int B, int Hq, int max_seq_len) {
    if (!valid_desc(desc) || B < 0 || Hq < 1 || max_seq_len < 0) return 0;
    tq::Layout L;
    tq::make_layout(*desc, &L);
    tq::AttnShape s{};
    s.n_seq = B;
    s.Hq = Hq;
    s.max_len = max_seq_len;
    s.is_decode = 1;
    return tq::attn_ws_bytes(L, s);
}

extern "C" int tq_decode_attn(const tq_params *kp, const tq_params *vp, const tq_cache_desc *desc, const void *Q,
                              int B, int Hq, const int32_t *block_table, int max_blocks, const int32_t *seq_lens,
                              int max_seq_len, const void *cache, int64_t num_blocks, void *out, float *lse,
                              float *logits, int64_t logits_stride, void *workspace, size_t workspace_bytes,
                              void *stream) {
    if (!attn_params_ok(kp, vp, desc, Hq)) {
        if (valid_desc(desc) && (desc->d > 256 || (Hq >= 1 && Hq % desc->n_kv_heads == 0 &&
                                                   Hq / desc->n_kv_heads > 8)))
            return TQ_EUNSUPPORTED;
        return TQ_EINVAL;
    }
    if (B < 0 || max_blocks < 0 || max_seq_len < 0 || num_blocks < 0) return TQ_EINVAL;
    if (B == 0) return TQ_OK;
    if (!Q || !block_table || !seq_lens || !cache || !out || !workspace) return TQ_EINVAL;
    if (!aligned(Q, 16) || !aligned(cache, 256) || !aligned(workspace, 256) || !aligned(out, 16)) return TQ_EINVAL;
    if (logits && logits_stride < max_seq_len) return TQ_EINVAL;
    if (int64_t(max_blocks) * desc->page_tokens < max_seq_len) return TQ_EINVAL;
    tq::Layout L;
    tq::make_layout(*desc, &L);
    tq::AttnShape s{};
    s.n_seq = B;
    s.Hq = Hq;
    s.block_table = block_table;
    s.bt_stride = max_blocks;
    s.max_blocks = max_blocks;
    s.seq_lens = seq_lens;
    s.is_decode = 1;
    s.base_len = 0;
    s.max_len = max_seq_len;
    if (workspace_bytes < tq::attn_ws_bytes(L, s)) return TQ_EINVAL;
    return cuda_status(tq::launch_attention(kp, vp, L, Q, s, static_cast<const uint8_t *>(cache), num_blocks, out,
                                            lse, logits, logits_stride, static_cast<uint8_t *>(workspace),
                                            workspace_bytes, stream));
}

extern "C" int tq_decode_step(const tq_params *kp, const tq_params *vp, const tq_cache_desc *desc, const void *K_new,
                              const void *V_new, const int32_t *slot_mapping, const void *Q, int B, int Hq,
                              const int32_t *block_table, int max_blocks, const int32_t *seq_lens, int max_seq_len,
                              void *cache, int64_t num_blocks, void *out, float *lse, float *logits,
                              int64_t logits_stride, void *workspace, size_t workspace_bytes, void *stream) {
    if (!attn_params_ok(kp, vp, desc, Hq)) {
        if (valid_desc(desc) && (desc->d > 256 || (Hq >= 1 && Hq % desc->n_kv_heads == 0 &&
                                                   Hq / desc->n_kv_heads > 8)))
            return TQ_EUNSUPPORTED;
        return TQ_EINVAL;
    }
    if (B < 0 || max_blocks < 0 || max_seq_len < 0 || num_blocks < 0) return TQ_EINVAL;
    if (B == 0) return TQ_OK;
    if (!K_new || !V_new || !slot_mapping || !Q || !block_table || !seq_lens || !cache || !out || !workspace)
        return TQ_EINVAL;
    if (!aligned(K_new, 16) || !aligned(V_new, 16) || !aligned(Q, 16) || !aligned(cache, 256) ||
        !aligned(workspace, 256) || !aligned(out, 16))
        return TQ_EINVAL;
    if (logits && logits_stride < max_seq_len) return TQ_EINVAL;
    if (int64_t(max_blocks) * desc->page_tokens < max_seq_len) return TQ_EINVAL;
    tq::Layout L;
    tq::make_layout(*desc, &L);
    tq::AttnShape s{};
    s.n_seq = B;
    s.Hq = Hq;
    s.block_table = block_table;
    s.bt_stride = max_blocks;
    s.max_blocks = max_blocks;
    s.seq_lens = seq_lens;
    s.is_decode = 1;
    s.base_len = 0;
    s.max_len = max_seq_len;
    if (workspace_bytes < tq::attn_ws_bytes(L, s)) return TQ_EINVAL;
    tq::StepTokens step{K_new, V_new, slot_mapping, static_cast<uint8_t *>(cache)};
    return cuda_status(tq::launch_attention(kp, vp, L, Q, s, static_cast<const uint8_t *>(cache), num_blocks, out,
                                            lse, logits, logits_stride, static_cast<uint8_t *>(workspace),
                                            workspace_bytes, stream, &step));
}

extern "C" size_t tq_prefill_workspace_bytes(const tq_cache_desc *desc, int C, int Hq, int seq_len) {
    if (!valid_desc(desc) || C < 0 || Hq < 1 || seq_len < C) return 0;
    tq::Layout L;
    tq::make_layout(*desc, &L);
    tq::AttnShape s{};
    s.n_seq = C;
    s.Hq = Hq;
    s.max_len = seq_len;
    return tq::attn_ws_bytes(L, s);
}

extern "C" int tq_prefill_attn(const tq_params *kp, const tq_params *vp, const tq_cache_desc *desc, const void *Q,
                               int C, int Hq, const int32_t *block_table, int max_blocks, int seq_len,
                               const void *cache, int64_t num_blocks, void *out, float *lse, void *workspace,
                               size_t workspace_bytes, void *stream) {
    if (!attn_params_ok(kp, vp, desc, Hq)) {
        if (valid_desc(desc) && desc->d > 256) return TQ_EUNSUPPORTED;
        return TQ_EINVAL;
    }
    if (C < 0 || seq_len < C || max_blocks < 0 || num_blocks < 0) return TQ_EINVAL;
    if (C == 0) return TQ_OK;
    if (!Q || !block_table || !cache || !out || !workspace) return TQ_EINVAL;
    if (!aligned(Q, 16) || !aligned(cache, 256) || !aligned(workspace, 256) || !aligned(out, 16)) return TQ_EINVAL;
    if (int64_t(max_blocks) * desc->page_tokens < seq_len) return TQ_EINVAL;
    tq::Layout L;
    tq::make_layout(*desc, &L);
    tq::AttnShape s{};
    s.n_seq = C;
    s.Hq = Hq;
    s.block_table = block_table;
    s.bt_stride = 0;
    s.max_blocks = max_blocks;
    s.seq_lens = nullptr;
    s.base_len = seq_len - C;
    s.max_len = seq_len;
    if (workspace_bytes < tq::attn_ws_bytes(L, s)) return TQ_EINVAL;
    return cuda_status(tq::launch_attention(kp, vp, L, Q, s, static_cast<const uint8_t *>(cache), num_blocks, out,
                                            lse, nullptr, 0, static_cast<uint8_t *>(workspace), workspace_bytes,
                                            stream));
}

extern "C" size_t tq_score_workspace_bytes(const tq_cache_desc *desc, int64_t n_db, int n_q, int k) {
    if (!valid_desc(desc) || n_db < 0 || n_q < 0 || k < 1 || k > 64) return 0;
    tq::Layout L;
    tq::make_layout(*desc, &L);
    return tq::score_ws_bytes(L, n_db, n_q, k);
}

extern "C" int tq_score(const tq_params *p, const tq_cache_desc *desc, const void *db_cache, int64_t n_db,
                        const float *Q, int n_q, int k, float *top_scores, int64_t *top_idx, void *workspace,
                        size_t workspace_bytes, void *stream) {
    if (!valid_desc(desc) || !p) return TQ_EINVAL;
    if (desc->n_kv_heads != 1 || desc->vbits != 0) return TQ_EINVAL;
    if (desc->kbits == 8 || desc->kbits == TQ_BITS_POLAR) return TQ_EUNSUPPORTED;
    if (p->d != desc->d || p->bits != desc->kbits) return TQ_EINVAL;
    if (n_db < 1 || n_q < 0 || k < 1 || k > 64 || k > n_db) return TQ_EINVAL;
    if (n_q == 0) return TQ_OK;
    if (!db_cache || !Q || !top_scores || !top_idx || !workspace) return TQ_EINVAL;
    if (!aligned(Q, 16) || !aligned(db_cache, 256) || !aligned(workspace, 256)) return TQ_EINVAL;
    tq::Layout L;
    tq::make_layout(*desc, &L);
    if (workspace_bytes < tq::score_ws_bytes(L, n_db, n_q, k)) return TQ_EINVAL;
    return cuda_status(tq::launch_score(p, L, static_cast<const uint8_t *>(db_cache), n_db, Q, n_q, k, top_scores,
                                        top_idx, static_cast<uint8_t *>(workspace), workspace_bytes, stream));
}

extern "C" int tq_read_status(void *workspace, void *stream, uint32_t *flags) {
    if (!workspace || !flags) return TQ_EINVAL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return TQ_ECUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return TQ_ECUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), st) != cudaSuccess) return TQ_ECUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return TQ_ECUDA;
    *flags = v;
    return TQ_OK;
}

extern "C" const char *tq_status_string(int status) {
    switch (status) {
        case TQ_OK: return "ok";
        case TQ_EINVAL: return "invalid argument";
        case TQ_EUNSUPPORTED: return "unsupported configuration";
        case TQ_ECUDA: return "CUDA error";
        case TQ_EDEVICE: return "device-side error flagged in the workspace status word";
        case TQ_ENOMEM: return "out of memory";
        case TQ_ESCRATCH: return "problem needs more scratch than the no-allocation entry point's static array";
    }
    return "unknown status";
}
