// Internal declarations shared by the libtqkv translation units.
// Host + device.  Nothing here is part of the C ABI (see include/tqkv.h).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "tqkv.h"

#if defined(__CUDACC__)
#define TQ_HD __host__ __device__
#else
#define TQ_HD
#endif

namespace tq {

// Byte layout of one page (page_tokens slots of one KV head).  Offsets are
// within the page; *_bpt are bytes per token of that field; -1 = absent.
// Field order and sizes follow the description in tqkv.h.
struct Layout {
    int d, kbits, kqjl, vbits, P, H;
    int kc_off, kc_bpt, kc_w;   // main K code array and its field width
    int kh_off, kh_bpt;         // K sign-bit array (3-bit codes only)
    int ks_off, ks_bpt;         // QJL sign bits
    int kn_off, kr_off;         // fp16 norms
    int vc_off, vc_bpt, vc_w;
    int vh_off, vh_bpt;
    int vn_off;
    int page_bytes;
    // Fractional rates (TQ_BITS_HALF | b): kc/kh above hold coordinates
    // 0 .. d/2-1 at ka_bits = b + 1 bits, kc2/kh2 coordinates d/2 .. d-1 at
    // kb_bits = b (likewise for values); ka_bits = kb_bits = kbits otherwise.
    int khalf, ka_bits, kb_bits, kc2_off, kc2_bpt, kc2_w, kh2_off, kh2_bpt;
    int vhalf, va_bits, vb_bits, vc2_off, vc2_bpt, vc2_w, vh2_off, vh2_bpt;
    // Polar codes (TQ_BITS_POLAR): kc holds the d/2 level-1 angle codes
    // (4 bits), kc2 the d/2 - 1 higher-level codes (2 bits, d/2 slots).
    int kpolar, vpolar;
};

inline bool is_half(int bits) { return (bits & TQ_BITS_HALF) != 0; }

inline int pad16(int x) { return (x + 15) & ~15; }

// Returns false if the description is invalid.
inline bool make_layout(const tq_cache_desc &c, Layout *L) {
    L->d = c.d; L->kbits = c.kbits; L->kqjl = c.kqjl; L->vbits = c.vbits;
    L->P = c.page_tokens; L->H = c.n_kv_heads;
    const int d = c.d, P = c.page_tokens;
    int off = 0;
    auto add = [&](int bpt, int *o, int *b) { *o = off; *b = bpt; off += pad16(P * bpt); };
    int dummy;
    L->kh_off = L->kh_bpt = L->ks_off = L->ks_bpt = L->kr_off = -1;
    L->vc_off = L->vc_bpt = L->vh_off = L->vh_bpt = L->vn_off = -1;
    L->vc_w = 0;
    L->kc2_off = L->kc2_bpt = L->kh2_off = L->kh2_bpt = -1;
    L->vc2_off = L->vc2_bpt = L->vh2_off = L->vh2_bpt = -1;
    L->kc2_w = L->vc2_w = 0;
    // one code of `bits` bits over n coordinates: a main array (w bits) and,
    // for 3 bits, a 2-bit array followed by a 1-bit sign array
    auto code = [&](int bits, int n, int *co, int *cb, int *cw, int *ho, int *hb) {
        if (bits == 8) { add(n, co, cb); *cw = 8; }
        else if (bits == 3) { add(n * 2 / 8, co, cb); *cw = 2; add(n / 8, ho, hb); }
        else { add(n * bits / 8, co, cb); *cw = bits; }
    };
    L->kpolar = c.kbits == TQ_BITS_POLAR ? 1 : 0;
    L->vpolar = c.vbits == TQ_BITS_POLAR ? 1 : 0;
    auto polar_codes = [&](int *co, int *cb, int *cw, int *c2o, int *c2b, int *c2w) {
        add(d / 2 * 4 / 8, co, cb); *cw = 4;
        add(d / 2 * 2 / 8, c2o, c2b); *c2w = 2;
    };
    L->khalf = is_half(c.kbits) ? 1 : 0;
    L->ka_bits = L->khalf ? (c.kbits & 7) + 1 : c.kbits;
    L->kb_bits = L->khalf ? (c.kbits & 7) : c.kbits;
    const int kn = L->khalf ? d / 2 : d;
    if (L->kpolar) {
        polar_codes(&L->kc_off, &L->kc_bpt, &L->kc_w, &L->kc2_off, &L->kc2_bpt, &L->kc2_w);
    } else {
        code(L->ka_bits, kn, &L->kc_off, &L->kc_bpt, &L->kc_w, &L->kh_off, &L->kh_bpt);
        if (L->khalf) code(L->kb_bits, d / 2, &L->kc2_off, &L->kc2_bpt, &L->kc2_w, &L->kh2_off, &L->kh2_bpt);
    }
    if (c.kqjl) add(d / 8, &L->ks_off, &L->ks_bpt);
    add(2, &L->kn_off, &dummy);
    if (c.kqjl) add(2, &L->kr_off, &dummy);
    L->vhalf = is_half(c.vbits) ? 1 : 0;
    L->va_bits = L->vhalf ? (c.vbits & 7) + 1 : c.vbits;
    L->vb_bits = L->vhalf ? (c.vbits & 7) : c.vbits;
    if (c.vbits > 0) {
        const int vn = L->vhalf ? d / 2 : d;
        if (L->vpolar) {
            polar_codes(&L->vc_off, &L->vc_bpt, &L->vc_w, &L->vc2_off, &L->vc2_bpt, &L->vc2_w);
        } else {
            code(L->va_bits, vn, &L->vc_off, &L->vc_bpt, &L->vc_w, &L->vh_off, &L->vh_bpt);
            if (L->vhalf) code(L->vb_bits, d / 2, &L->vc2_off, &L->vc2_bpt, &L->vc2_w, &L->vh2_off, &L->vh2_bpt);
        }
        add(2, &L->vn_off, &dummy);
    }
    L->page_bytes = off;
    return true;
}

// Library-owned parameters.  Device arrays live in one allocation.
struct DevParams {
    int d, bits;
    const float *signs;      // [d] +1/-1
    const uint16_t *S;       // [d][d] bf16 bits, row-major (row j = projection j)
    const uint16_t *S16;     // the same matrix as fp16 bits (exact for |S| >= 2^-14)
    const float *lv;         // [2^bits] levels indexed by the stored sign-magnitude code
    const float *bounds;     // [2^bits - 1] ascending decision boundaries
    // fractional rates: lv / bounds belong to the (b + 1)-bit codebook of
    // coordinates 0 .. d/2-1, lv2 / bounds2 to the b-bit one of the rest
    const float *lv2, *bounds2;
    // polar codes (TQ_BITS_POLAR): level-1 bounds [0, 16), cos / sin of the
    // level-1 centres [16, 32) / [32, 48), level l >= 2 at 48 + 12 (l - 2):
    // 3 bounds, 4 cos, 4 sin of its centres; cos / sin of the level-1 bounds
    // 0 .. 6 at 136 + 2j, of the level-l bounds at 152 + 6 (l - 2) + 2j
    const float *polar;
    // d == 128 only (else null): 32 KB images of 128 x 128 operand tiles laid
    // out exactly as the tensor cores read them from shared memory (K-major,
    // 128-byte swizzle, two 64-column halves), so one bulk copy stages them.
    const uint8_t *rot_img;  // bf16 (H D)[n][k] = (-1)^popcount(n & k) * D[k]
    const uint8_t *s16_img;  // fp16 S[n][k] (exact for |S| >= 2^-17)
    // Dense random rotation (rot = 1, d <= 256) instead of H D / sqrt(d):
    // Rd[j][i] (y = Rd x) and its transpose RdT (x = Rd^T y), fp32.
    int rot;
    const float *Rd, *RdT;
    // Magnitude cells of a 1- to 4-bit codebook (null for fractional rates,
    // polar codes, or when the thresholds are too close): with x = cellC |u|
    // (cellC a power of two, so the scaled thresholds X_k are exact), cell
    // c = min(floor(x), 15) holds at most one X_k; entry c is {X in the cell
    // (else 3e38), #{X_k <= c} as int bits, |level| of that rank, |level| of
    // the next}.  The magnitude rank is #{X_k <= x}.
    const float4 *cells;
    float cellC;
};

// Byte offset of element (row, col) of a 128 x 128 16-bit tile in the
// 128-byte-swizzled K-major image: column half col / 64 at 16 KB, rows of 128
// bytes, the 16-byte piece index XORed with row % 8.
inline size_t sw128_image_offset(int row, int col) {
    const int half = col >> 6, c = col & 63;
    const int piece = c >> 3, e = c & 7;
    return size_t(half) * 16384 + size_t(row) * 128 + size_t(((piece ^ (row & 7)) << 4) + e * 2);
}

}  // namespace tq

struct tq_params {
    int d, bits;
    uint64_t seed;
    int device;
    int8_t *h_signs;         // host copies
    float *h_S;
    float *h_levels;         // ascending bucket order
    float *h_bounds;
    float *h_R;              // dense rotation [d][d] (nullptr: H D / sqrt(d))
    void *d_block;           // device allocation
    tq::DevParams dev;
};

namespace tq {

// Workspace header: the first 256 bytes of every workspace.
constexpr size_t kWsHeader = 256;

// Launchers (defined in the .cu files).  Return cudaError_t as int.
int launch_encode(const tq_params *kp, const tq_params *vp, const Layout &L, const void *K,
                  const void *V, int in_dtype, int64_t n_tokens, const int32_t *slots,
                  uint8_t *cache, int64_t num_blocks, uint8_t *ws, size_t ws_bytes, void *stream);
size_t encode_ws_bytes(const Layout &L, int64_t n_tokens);
// Fused d = 128 bf16 encoder; returns -1 when the configuration is not covered.
int launch_encode128(const tq_params *kp, const tq_params *vp, const Layout &L, const void *K, const void *V,
                     int64_t n_tokens, const int32_t *slots, uint8_t *cache, int64_t num_blocks, uint8_t *ws,
                     void *stream);

struct AttnShape {
    int n_seq;            // decode: batch; prefill: chunk length C
    int Hq;
    const int32_t *block_table;
    int bt_stride;        // decode: max_blocks; prefill: 0 (all rows share one table)
    int max_blocks;
    const int32_t *seq_lens;   // decode: [B]; prefill: nullptr
    int base_len;         // prefill: seq_len - C (query j sees base_len + j + 1)
    int max_len;          // longest visible length
    int is_decode;        // 1: decode (per-sequence lengths), 0: prefill chunk
};
// New tokens of a fused decode step (one per sequence): bf16 K and V
// [B][H][d], their slots, and the cache they are written into.
struct StepTokens {
    const void *K, *V;
    const int32_t *slots;
    uint8_t *cache;
};
size_t attn_ws_bytes(const Layout &L, const AttnShape &s);
int launch_attention(const tq_params *kp, const tq_params *vp, const Layout &L, const void *Q,
                     const AttnShape &s, const uint8_t *cache, int64_t num_blocks, void *out,
                     float *lse, float *logits, int64_t logits_stride, uint8_t *ws,
                     size_t ws_bytes, void *stream, const StepTokens *step = nullptr);

// Testing aid of the tensor-core decode kernel: the poll budget of a wait
// that nothing completes, taken (and reset to 0) by the next launch.
uint32_t take_decode_stall();
void set_decode_stall(uint32_t polls);

// Blocks of the tensor-core decode kernel resident per SM (0: not covered).
int dec128_resident(const Layout &L, int G);

// Tensor-core attention for d = 128 (decode and prefill query groups);
// returns -1 when the configuration is not covered.
int launch_dec128(const tq_params *kp, const tq_params *vp, const Layout &L, const float *qr, const float *w,
                  const AttnShape &s, int G, int n_groups, int n_splits, int split_len, const uint8_t *cache,
                  int64_t num_blocks, float *part_o, float *part_ml, float *logits, int64_t logits_stride,
                  uint32_t *status, cudaStream_t st);

// w[r] = S q_r[r] for rows x D fp32 rows (S as bf16 bits, row j = projection j).
int launch_qproj(const float *qr, int64_t rows, int D, const uint16_t *S, float *w, cudaStream_t st);

// Tensor-core chunked prefill for d = 128, 64-token pages, b-bit + QJL keys
// and b-bit values (b in 2..4), 128 % G == 0: whether it applies, its key
// split (count, length in keys), and the launcher writing combine partials.
bool pf128_covers(const Layout &L, const AttnShape &s);
int pf128_splits(const Layout &L, const AttnShape &s, int *split_len);
int launch_pf128(const tq_params *kp, const tq_params *vp, const Layout &L, const float *qr, const float *w,
                 const AttnShape &s, int n_splits, int split_len, const uint8_t *cache, int64_t num_blocks,
                 float *part_o, float *part_ml, uint32_t *status, cudaStream_t st);

size_t score_ws_bytes(const Layout &L, int64_t n_db, int n_q, int k);
// Tensor-core search (4-bit + QJL database, d in {128, 256, 512, 1024},
// k <= 16): blocks per query tile, or 0 when not covered; workspace pieces;
// launcher of the query-feature and scoring kernels (writes 2 * n_groups
// candidate lists per query into pv / pi).
int search_tc_groups(const Layout &L, int64_t n_db, int n_q, int k);
size_t search_tc_qf_bytes(const Layout &L, int n_q);
size_t search_tc_qscale_bytes(int n_q);
int launch_search_tc(const tq_params *p, const Layout &L, const uint8_t *db, int64_t n_db, int n_q, int k,
                     const float *qr, const float *w, uint8_t *qf, float *qscale, float *pv, int64_t *pi,
                     int n_groups, uint32_t *status, cudaStream_t st);
int launch_score(const tq_params *p, const Layout &L, const uint8_t *db, int64_t n_db,
                 const float *Q, int n_q, int k, float *top_scores, int64_t *top_idx,
                 uint8_t *ws, size_t ws_bytes, void *stream);

}  // namespace tq
