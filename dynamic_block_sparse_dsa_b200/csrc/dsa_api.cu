// dsa_api.cu -- the C ABI (include/dsa.h): host-side validation, workspace
// sizing and launches on the caller's stream.  No allocation, no host sync.
#include <climits>
#include <cstdint>

#include "dsa_kernels.h"

namespace {

using namespace dsa;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// log2 of a supported block size (64, 128, 256, 512 tokens), or -1
int block_shift_of(int block_size) {
    for (int sh = kMinBlockShift; sh <= kMaxBlockShift; ++sh)
        if (block_size == (1 << sh)) return sh;
    return -1;
}

int check_cache(const dsa_kv_cache *c) {
    if (!c || !c->k_pool || !c->v_pool || !c->kc_pool) return DSA_ERR_INVALID_ARG;
    if (!aligned16(c->k_pool) || !aligned16(c->v_pool) || !aligned16(c->kc_pool)) return DSA_ERR_INVALID_ARG;
    if (c->num_pages < 1 || c->num_kv_heads < 1) return DSA_ERR_INVALID_ARG;
    if (block_shift_of(c->block_size) < 0 || c->head_dim != kHeadDim || c->idx_dim != kIdxDim)
        return DSA_ERR_UNSUPPORTED;
    return DSA_OK;
}

int check_seqs(const dsa_seqs *s) {
    if (!s || !s->block_table || !s->seq_lens) return DSA_ERR_INVALID_ARG;
    if (s->num_seqs < 1 || s->max_blocks < 1) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

int check_queries(const dsa_queries *q) {
    if (!q || q->total_q < 0) return DSA_ERR_INVALID_ARG;
    if (q->total_q > 0 && (!q->cu_q || !q->q_pos)) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

int sm_count() {
    static int cached[64] = {};
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev >= 0 && dev < 64) cached[dev] = n;
    return n;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// decode workspace: [split counters int32 T*Hkv][partials f32 2*kAttnMaxCtas*G*kAttnPartStride]
struct DecodeLayout {
    size_t counters, part, total;
};
DecodeLayout decode_layout(int total_q, int hq, int hkv) {
    DecodeLayout L;
    L.counters = 0;
    L.part = align_up((size_t)total_q * hkv * sizeof(int32_t), 256);
    L.total = align_up(L.part + (size_t)2 * kAttnMaxCtas * (hq / hkv) * kAttnPartStride * sizeof(float), 256);
    return L;
}

// select workspace: [counters int32 T][candidate keys u64 T*kSelMaxChunks*(kSelMaxK-1)]
struct SelectLayout {
    size_t counters, cand, total;
};
SelectLayout select_layout(int total_q) {
    SelectLayout L;
    L.counters = 0;
    L.cand = align_up((size_t)total_q * sizeof(int32_t), 256);
    L.total = align_up(L.cand + (size_t)total_q * kSelMaxChunks * (kSelMaxK - 1) * sizeof(unsigned long long), 256);
    return L;
}

// single-launch decode workspace: [header 256 B][sel_count T][flags T]
// [split counters T*Hkv][candidates kAttnMaxCtas*2*(kSelMaxK-1) u64][partials]
struct FusedLayout {
    size_t hdr, sel_count, flags, counters, cand, part, total;
};
FusedLayout fused_layout(int total_q, int hq, int hkv) {
    FusedLayout L;
    L.hdr = 0;
    L.sel_count = 256;
    L.flags = align_up(L.sel_count + (size_t)total_q * 4, 256);
    L.counters = align_up(L.flags + (size_t)total_q * 4, 256);
    L.cand = align_up(L.counters + (size_t)total_q * hkv * 4, 256);
    L.part = align_up(L.cand + (size_t)kAttnMaxCtas * 2 * (kSelMaxK - 1) * sizeof(unsigned long long), 256);
    L.total = align_up(L.part + (size_t)2 * kAttnMaxCtas * (hq / hkv) * kAttnPartStride * sizeof(float), 256);
    return L;
}

// grid of the persistent attention kernel: one CTA per SM, never more CTAs
// than work items so that every CTA owns a non-empty range
void attn_schedule(AttnArgs &a, bool allow_split, bool allow_cluster = false) {
    const long long pairs = (long long)a.total_q * a.num_kv_heads;
    a.total_units = (pairs * a.k_max) << a.tile_shift;
    long long C = sm_count();
    if (C > kAttnMaxCtas) C = kAttnMaxCtas;
    a.cluster2 = 0;
    a.interleave = 0;
    // between a quarter and a half as many pairs as SMs: one 2-CTA cluster per
    // pair keeps at least half of the SMs streaming and merges on chip
    if (allow_cluster && allow_split && (a.k_max << a.tile_shift) >= 2 && 4 * pairs >= C && 2 * pairs <= C) {
        a.cluster2 = 1;
        a.pair_aligned = 0;
        a.num_ctas = (int)(2 * pairs);
        return;
    }
    // whole (query, KV head) pairs per CTA when there are plenty of them (or
    // when no workspace is available); otherwise split pairs across CTAs
    a.pair_aligned = (!allow_split || pairs >= 16 * C) ? 1 : 0;
    const long long items = a.pair_aligned ? pairs : a.total_units;
    if (C > items) C = items;
    // a pair may be split over at most ~60 CTAs (the kernel merges <= 63 partials)
    if (C > pairs * 60) C = pairs * 60;
    a.num_ctas = (int)C;
    // whole pairs: KV-head-major and interleaved over the CTAs (a query's
    // selected blocks are scattered over the pool, so the queries running at
    // one time share blocks only through L2, and one KV head's slice of the
    // pool fits there where the whole pool often does not)
    a.interleave = (a.pair_aligned && a.num_kv_heads > 1) ? 1 : 0;
}

int attn_common(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                const void *q, int32_t num_q_heads, const int32_t *sel, const int32_t *cnt,
                int32_t k_max, float sm_scale, void *out, float *lse, int32_t *dev_err, AttnArgs &a) {
    int rc;
    if ((rc = check_cache(cache)) || (rc = check_seqs(seqs)) || (rc = check_queries(queries))) return rc;
    if (queries->total_q > 0 && (!q || !sel || !cnt || !out)) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out) || !aligned16(sel)) return DSA_ERR_INVALID_ARG;
    if (k_max < 1 || num_q_heads < 1) return DSA_ERR_INVALID_ARG;
    if (num_q_heads % cache->num_kv_heads != 0) return DSA_ERR_INVALID_ARG;
    const int group = num_q_heads / cache->num_kv_heads;
    if (group > kMaxGroup) return DSA_ERR_UNSUPPORTED;
    if (!(sm_scale > 0.f)) return DSA_ERR_INVALID_ARG;
    // TMA coordinates are int32: pool rows (page*64+token) and query rows (t*Hq+h);
    // work units (query, KV head, selection slot) are counted in 32 bits
    const int bsh = block_shift_of(cache->block_size);
    if (((long long)cache->num_pages << bsh) >= (1LL << 31) ||
        (long long)queries->total_q * num_q_heads >= (1LL << 31) ||
        (((long long)queries->total_q * cache->num_kv_heads * k_max) << (bsh - 6)) >= (1LL << 31))
        return DSA_ERR_UNSUPPORTED;
    a = AttnArgs{};
    a.block_shift = bsh;
    a.tile_shift = bsh - 6;
    a.k_pool = static_cast<const __nv_bfloat16 *>(cache->k_pool);
    a.v_pool = static_cast<const __nv_bfloat16 *>(cache->v_pool);
    a.num_pages = cache->num_pages;
    a.num_kv_heads = cache->num_kv_heads;
    a.block_table = seqs->block_table;
    a.max_blocks = seqs->max_blocks;
    a.seq_lens = seqs->seq_lens;
    a.num_seqs = seqs->num_seqs;
    a.cu_q = queries->cu_q;
    a.q_pos = queries->q_pos;
    a.total_q = queries->total_q;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.num_q_heads = num_q_heads;
    a.group = group;
    a.sel = sel;
    a.cnt = cnt;
    a.k_max = k_max;
    a.scale_log2 = sm_scale * 1.4426950408889634f;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.dev_err = dev_err;
    return DSA_OK;
}

int select_common(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                  const int8_t *q_idx, const int32_t *w, int32_t num_idx_heads, int32_t w_abs_max,
                  const int32_t *k_per_seq, int32_t k_max, int32_t *sel, int32_t *cnt, void *workspace,
                  size_t workspace_bytes, const KvAppendArgs *app, int32_t *dev_err, dsa_stream_t stream);

int wide_common(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries, const void *q_idx,
                const int32_t *w, int32_t num_idx_heads, int64_t *scores, int32_t *dev_err, IndexScoreArgs &a) {
    int rc;
    if ((rc = check_cache(cache)) || (rc = check_seqs(seqs)) || (rc = check_queries(queries))) return rc;
    if (num_idx_heads < 1) return DSA_ERR_INVALID_ARG;
    if (num_idx_heads > kMaxIdxHeads) return DSA_ERR_UNSUPPORTED;
    if (queries->total_q > 0 && (!q_idx || !w || !scores || !aligned16(q_idx))) return DSA_ERR_INVALID_ARG;
    a = IndexScoreArgs{};
    a.block_shift = block_shift_of(cache->block_size);
    a.kc_pool = cache->kc_pool;
    a.num_pages = cache->num_pages;
    a.block_table = seqs->block_table;
    a.max_blocks = seqs->max_blocks;
    a.seq_lens = seqs->seq_lens;
    a.num_seqs = seqs->num_seqs;
    a.cu_q = queries->cu_q;
    a.q_pos = queries->q_pos;
    a.total_q = queries->total_q;
    a.q_idx = static_cast<const int8_t *>(q_idx);
    a.w = w;
    a.num_idx_heads = num_idx_heads;
    a.scores = nullptr;
    a.dev_err = dev_err;
    return DSA_OK;
}

}  // namespace

namespace dsa {
int check_decode_attn_args(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                           const void *q, int32_t num_q_heads, const int32_t *sel, const int32_t *cnt,
                           int32_t k_max, float sm_scale, void *out, float *lse) {
    AttnArgs a;
    return attn_common(cache, seqs, queries, q, num_q_heads, sel, cnt, k_max, sm_scale, out, lse, nullptr, a);
}
}  // namespace dsa

extern "C" {

int dsa_version(void) { return 100; }

const char *dsa_status_string(int status) {
    switch (status) {
        case DSA_OK: return "ok";
        case DSA_ERR_INVALID_ARG: return "invalid argument";
        case DSA_ERR_UNSUPPORTED: return "unsupported size";
        case DSA_ERR_RANGE: return "int32 score range exceeded";
        case DSA_ERR_WORKSPACE: return "workspace too small";
        case DSA_ERR_CUDA: return "CUDA error";
        default: return "unknown status";
    }
}

int dsa_kv_append(const dsa_kv_cache *cache, const dsa_seqs *seqs, const int32_t *cu_new,
                  int32_t total_new, const void *k_new, const void *v_new, const int8_t *kc_new,
                  int32_t *dev_err, dsa_stream_t stream) {
    int rc;
    if ((rc = check_cache(cache)) || (rc = check_seqs(seqs))) return rc;
    if (total_new < 0) return DSA_ERR_INVALID_ARG;
    if (total_new == 0) return DSA_OK;
    if (!cu_new || !k_new || !v_new) return DSA_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || (kc_new && !aligned16(kc_new))) return DSA_ERR_INVALID_ARG;
    KvAppendArgs a{};
    a.block_shift = block_shift_of(cache->block_size);
    a.k_pool = cache->k_pool;
    a.v_pool = cache->v_pool;
    a.kc_pool = cache->kc_pool;
    a.num_pages = cache->num_pages;
    a.num_kv_heads = cache->num_kv_heads;
    a.block_table = seqs->block_table;
    a.max_blocks = seqs->max_blocks;
    a.seq_lens = seqs->seq_lens;
    a.num_seqs = seqs->num_seqs;
    a.cu_new = cu_new;
    a.total_new = total_new;
    a.k_new = k_new;
    a.v_new = v_new;
    a.kc_new = kc_new;
    a.dev_err = dev_err;
    return from_cuda(launch_kv_append(a, reinterpret_cast<cudaStream_t>(stream)));
}

int dsa_index_score(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                    const int8_t *q_idx, const int32_t *w, int32_t num_idx_heads, int32_t w_abs_max,
                    int32_t *scores, int32_t *dev_err, dsa_stream_t stream) {
    int rc;
    if ((rc = check_cache(cache)) || (rc = check_seqs(seqs)) || (rc = check_queries(queries))) return rc;
    if (num_idx_heads < 1 || w_abs_max < 0) return DSA_ERR_INVALID_ARG;
    if (num_idx_heads > kMaxIdxHeads) return DSA_ERR_UNSUPPORTED;
    // |S| <= H * |w| * idx_dim * 128 * 128 must stay below 2^31 for exact int32
    const long long bound = (long long)num_idx_heads * w_abs_max * kIdxDim * 128LL * 128LL;
    if (bound >= (1LL << 31)) return DSA_ERR_RANGE;
    if (queries->total_q == 0) return DSA_OK;
    if (!q_idx || !w || !scores || !aligned16(q_idx)) return DSA_ERR_INVALID_ARG;
    IndexScoreArgs a{};
    a.block_shift = block_shift_of(cache->block_size);
    a.kc_pool = cache->kc_pool;
    a.num_pages = cache->num_pages;
    a.block_table = seqs->block_table;
    a.max_blocks = seqs->max_blocks;
    a.seq_lens = seqs->seq_lens;
    a.num_seqs = seqs->num_seqs;
    a.cu_q = queries->cu_q;
    a.q_pos = queries->q_pos;
    a.total_q = queries->total_q;
    a.q_idx = q_idx;
    a.w = w;
    a.num_idx_heads = num_idx_heads;
    a.scores = scores;
    a.dev_err = dev_err;
    // prefill-shaped batches (on average a query tile per sequence) run on the
    // tensor cores; decode-shaped ones scan with dp4a (as do batches whose
    // positions array is not 16-byte aligned: the tensor-core kernel copies it
    // in 16-byte pieces)
    if ((long long)queries->total_q >= (long long)index_score_tc_min_queries_per_seq() * seqs->num_seqs &&
        aligned16(queries->q_pos))
        return from_cuda(launch_index_score_tc(a, sm_count(), reinterpret_cast<cudaStream_t>(stream)));
    return from_cuda(launch_index_score(a, reinterpret_cast<cudaStream_t>(stream)));
}

int dsa_topk_blocks(const dsa_seqs *seqs, const dsa_queries *queries, const int32_t *scores,
                    const int32_t *k_per_seq, int32_t k_max, int32_t block_size, int32_t *sel, int32_t *cnt,
                    int32_t *dev_err, dsa_stream_t stream) {
    int rc;
    if ((rc = check_seqs(seqs)) || (rc = check_queries(queries))) return rc;
    if (k_max < 1) return DSA_ERR_INVALID_ARG;
    if (block_shift_of(block_size) < 0) return DSA_ERR_UNSUPPORTED;
    if (k_max > kSelMaxK || seqs->max_blocks > topk_max_blocks()) return DSA_ERR_UNSUPPORTED;
    if (queries->total_q == 0) return DSA_OK;
    if (!scores || !k_per_seq || !sel || !cnt) return DSA_ERR_INVALID_ARG;
    TopkArgs a{};
    a.block_shift = block_shift_of(block_size);
    a.seq_lens = seqs->seq_lens;
    a.num_seqs = seqs->num_seqs;
    a.max_blocks = seqs->max_blocks;
    a.cu_q = queries->cu_q;
    a.q_pos = queries->q_pos;
    a.total_q = queries->total_q;
    a.scores = scores;
    a.k_per_seq = k_per_seq;
    a.k_max = k_max;
    a.sel = sel;
    a.cnt = cnt;
    a.dev_err = dev_err;
    return from_cuda(launch_topk(a, reinterpret_cast<cudaStream_t>(stream)));
}


int dsa_index_score_i64(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                        const int8_t *q_idx, const int32_t *w, int32_t num_idx_heads, int64_t *scores,
                        int32_t *dev_err, dsa_stream_t stream) {
    IndexScoreArgs a;
    int rc = wide_common(cache, seqs, queries, q_idx, w, num_idx_heads, scores, dev_err, a);
    if (rc || queries->total_q == 0) return rc;
    return from_cuda(launch_index_score_wide(a, false, scores, reinterpret_cast<cudaStream_t>(stream)));
}

int dsa_index_score_fp8(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                        const uint8_t *q_idx_e4m3, const int32_t *w, int32_t num_idx_heads, int32_t w_abs_max,
                        int64_t *scores, int32_t *dev_err, dsa_stream_t stream) {
    IndexScoreArgs a;
    int rc = wide_common(cache, seqs, queries, q_idx_e4m3, w, num_idx_heads, scores, dev_err, a);
    if (rc) return rc;
    if (w_abs_max < 0) return DSA_ERR_INVALID_ARG;
    // |S| * 2^18 <= H * |w| * 64 * (448 * 2^9)^2 must stay below 2^63
    const double bound = (double)num_idx_heads * w_abs_max * kIdxDim * (448.0 * 512.0) * (448.0 * 512.0);
    if (bound >= 9.2e18) return DSA_ERR_RANGE;
    if (queries->total_q == 0) return DSA_OK;
    return from_cuda(launch_index_score_wide(a, true, scores, reinterpret_cast<cudaStream_t>(stream)));
}

int dsa_topk_blocks_i64(const dsa_seqs *seqs, const dsa_queries *queries, const int64_t *scores,
                        const int32_t *k_per_seq, int32_t k_max, int32_t block_size, int32_t *sel,
                        int32_t *cnt, int32_t *dev_err, dsa_stream_t stream) {
    int rc;
    if ((rc = check_seqs(seqs)) || (rc = check_queries(queries))) return rc;
    if (k_max < 1) return DSA_ERR_INVALID_ARG;
    if (block_shift_of(block_size) < 0 || k_max > kSelMaxK) return DSA_ERR_UNSUPPORTED;
    if (queries->total_q == 0) return DSA_OK;
    if (!scores || !k_per_seq || !sel || !cnt) return DSA_ERR_INVALID_ARG;
    TopkArgs a{};
    a.block_shift = block_shift_of(block_size);
    a.seq_lens = seqs->seq_lens;
    a.num_seqs = seqs->num_seqs;
    a.max_blocks = seqs->max_blocks;
    a.cu_q = queries->cu_q;
    a.q_pos = queries->q_pos;
    a.total_q = queries->total_q;
    a.scores = nullptr;
    a.k_per_seq = k_per_seq;
    a.k_max = k_max;
    a.sel = sel;
    a.cnt = cnt;
    a.dev_err = dev_err;
    return from_cuda(launch_topk_wide(a, scores, reinterpret_cast<cudaStream_t>(stream)));
}

size_t dsa_select_blocks_workspace_size(int32_t total_q) {
    if (total_q <= 0) return 0;
    return select_layout(total_q).total;
}

int dsa_select_blocks(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                      const int8_t *q_idx, const int32_t *w, int32_t num_idx_heads, int32_t w_abs_max,
                      const int32_t *k_per_seq, int32_t k_max, int32_t *sel, int32_t *cnt, void *workspace,
                      size_t workspace_bytes, int32_t *dev_err, dsa_stream_t stream) {
    return select_common(cache, seqs, queries, q_idx, w, num_idx_heads, w_abs_max, k_per_seq, k_max, sel, cnt,
                         workspace, workspace_bytes, nullptr, dev_err, stream);
}

int dsa_select_blocks_append(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                             const int32_t *cu_new, int32_t total_new, const void *k_new, const void *v_new,
                             const int8_t *kc_new, const int8_t *q_idx, const int32_t *w, int32_t num_idx_heads,
                             int32_t w_abs_max, const int32_t *k_per_seq, int32_t k_max, int32_t *sel,
                             int32_t *cnt, void *workspace, size_t workspace_bytes, int32_t *dev_err,
                             dsa_stream_t stream) {
    int rc;
    if ((rc = check_cache(cache)) || (rc = check_seqs(seqs))) return rc;
    if (total_new < 0) return DSA_ERR_INVALID_ARG;
    if (total_new > 0) {
        if (!cu_new || !k_new || !v_new) return DSA_ERR_INVALID_ARG;
        if (!aligned16(k_new) || !aligned16(v_new) || (kc_new && !aligned16(kc_new))) return DSA_ERR_INVALID_ARG;
    }
    KvAppendArgs a{};
    a.block_shift = block_shift_of(cache->block_size);
    a.k_pool = cache->k_pool;
    a.v_pool = cache->v_pool;
    a.kc_pool = cache->kc_pool;
    a.num_pages = cache->num_pages;
    a.num_kv_heads = cache->num_kv_heads;
    a.block_table = seqs->block_table;
    a.max_blocks = seqs->max_blocks;
    a.seq_lens = seqs->seq_lens;
    a.num_seqs = seqs->num_seqs;
    a.cu_new = cu_new;
    a.total_new = total_new;
    a.k_new = k_new;
    a.v_new = v_new;
    a.kc_new = kc_new;
    a.dev_err = dev_err;
    a.overlap_prev = 0;
    // the append runs as extra CTAs of the selection's grid; with no queries
    // there is no selection launch, so it is launched on its own
    rc = select_common(cache, seqs, queries, q_idx, w, num_idx_heads, w_abs_max, k_per_seq, k_max, sel, cnt,
                       workspace, workspace_bytes, total_new > 0 ? &a : nullptr, dev_err, stream);
    if (rc || total_new == 0 || queries->total_q > 0) return rc;
    return from_cuda(launch_kv_append(a, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {
int select_common(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                  const int8_t *q_idx, const int32_t *w, int32_t num_idx_heads, int32_t w_abs_max,
                  const int32_t *k_per_seq, int32_t k_max, int32_t *sel, int32_t *cnt, void *workspace,
                  size_t workspace_bytes, const KvAppendArgs *app, int32_t *dev_err, dsa_stream_t stream) {
    int rc;
    if ((rc = check_cache(cache)) || (rc = check_seqs(seqs)) || (rc = check_queries(queries))) return rc;
    if (num_idx_heads < 1 || w_abs_max < 0 || k_max < 1) return DSA_ERR_INVALID_ARG;
    if (num_idx_heads > kMaxIdxHeads || k_max > kSelMaxK || seqs->max_blocks > kSelMaxChunks * 4096)
        return DSA_ERR_UNSUPPORTED;
    const long long bound = (long long)num_idx_heads * w_abs_max * kIdxDim * 128LL * 128LL;
    if (bound >= (1LL << 31)) return DSA_ERR_RANGE;
    if (queries->total_q == 0) return DSA_OK;
    if (!q_idx || !w || !k_per_seq || !sel || !cnt || !aligned16(q_idx)) return DSA_ERR_INVALID_ARG;
    const SelectLayout L = select_layout(queries->total_q);
    if (!workspace || !aligned16(workspace) || workspace_bytes < L.total) return DSA_ERR_WORKSPACE;
    SelectArgs a{};
    a.block_shift = block_shift_of(cache->block_size);
    a.kc_pool = cache->kc_pool;
    a.num_pages = cache->num_pages;
    a.block_table = seqs->block_table;
    a.max_blocks = seqs->max_blocks;
    a.seq_lens = seqs->seq_lens;
    a.num_seqs = seqs->num_seqs;
    a.cu_q = queries->cu_q;
    a.q_pos = queries->q_pos;
    a.total_q = queries->total_q;
    a.q_idx = q_idx;
    a.w = w;
    a.num_idx_heads = num_idx_heads;
    a.k_per_seq = k_per_seq;
    a.k_max = k_max;
    a.sel = sel;
    a.cnt = cnt;
    char *ws = static_cast<char *>(workspace);
    a.counters = reinterpret_cast<int32_t *>(ws + L.counters);
    a.cand = reinterpret_cast<unsigned long long *>(ws + L.cand);
    a.dev_err = dev_err;
    a.cu_new = app ? app->cu_new : nullptr;
    if (app) a.app = *app;
    return from_cuda(launch_select_blocks(a, reinterpret_cast<cudaStream_t>(stream)));
}
}  // namespace

extern "C" {

size_t dsa_sparse_attn_decode_workspace_size(int32_t total_q, int32_t num_q_heads, int32_t num_kv_heads,
                                             int32_t k_max) {
    if (total_q <= 0 || num_q_heads < 1 || num_kv_heads < 1 || k_max < 1 || num_q_heads % num_kv_heads)
        return 0;
    return decode_layout(total_q, num_q_heads, num_kv_heads).total;
}

int dsa_sparse_attn_decode(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                           const void *q, int32_t num_q_heads, const int32_t *sel, const int32_t *cnt,
                           int32_t k_max, float sm_scale, void *out, float *lse, void *workspace,
                           size_t workspace_bytes, int32_t *dev_err, dsa_stream_t stream) {
    AttnArgs a;
    int rc = attn_common(cache, seqs, queries, q, num_q_heads, sel, cnt, k_max, sm_scale, out, lse, dev_err, a);
    if (rc) return rc;
    if (queries->total_q == 0) return DSA_OK;
    const DecodeLayout L = decode_layout(queries->total_q, num_q_heads, cache->num_kv_heads);
    if (!workspace || !aligned16(workspace) || workspace_bytes < L.total) return DSA_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);
    a.counters = reinterpret_cast<int32_t *>(ws + L.counters);
    a.part = reinterpret_cast<float *>(ws + L.part);
    attn_schedule(a, true, true);
    return from_cuda(launch_sparse_attn(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t dsa_decode_fused_workspace_size(int32_t total_q, int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t k_max) {
    if (total_q <= 0 || num_q_heads < 1 || num_kv_heads < 1 || k_max < 1 || num_q_heads % num_kv_heads)
        return 0;
    return fused_layout(total_q, num_q_heads, num_kv_heads).total;
}

int dsa_decode_fused(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                     const int32_t *cu_new, int32_t total_new, const void *k_new, const void *v_new,
                     const int8_t *kc_new, const int8_t *q_idx, const int32_t *w, int32_t num_idx_heads,
                     int32_t w_abs_max, const int32_t *k_per_seq, int32_t k_max, const void *q,
                     int32_t num_q_heads, float sm_scale, int32_t *sel, int32_t *cnt, void *out, float *lse,
                     void *workspace, size_t workspace_bytes, int32_t *dev_err, dsa_stream_t stream) {
    AttnArgs a;
    int rc = attn_common(cache, seqs, queries, q, num_q_heads, sel, cnt, k_max, sm_scale, out, lse, dev_err, a);
    if (rc) return rc;
    if (num_idx_heads < 1 || w_abs_max < 0 || total_new < 0) return DSA_ERR_INVALID_ARG;
    if (num_idx_heads > kMaxIdxHeads || k_max > kSelMaxK || queries->total_q > kFusedMaxQ ||
        cache->block_size != kBlockSize)   // the single-launch step keeps 64-token blocks
        return DSA_ERR_UNSUPPORTED;
    const long long bound = (long long)num_idx_heads * w_abs_max * kIdxDim * 128LL * 128LL;
    if (bound >= (1LL << 31)) return DSA_ERR_RANGE;
    if (total_new > 0) {
        if (!cu_new || !k_new || !v_new) return DSA_ERR_INVALID_ARG;
        if (!aligned16(k_new) || !aligned16(v_new) || (kc_new && !aligned16(kc_new))) return DSA_ERR_INVALID_ARG;
    }
    if (queries->total_q == 0) return DSA_OK;
    if (!q_idx || !w || !k_per_seq || !aligned16(q_idx)) return DSA_ERR_INVALID_ARG;
    const FusedLayout L = fused_layout(queries->total_q, num_q_heads, cache->num_kv_heads);
    if (!workspace || !aligned16(workspace) || workspace_bytes < L.total) return DSA_ERR_WORKSPACE;
    char *ws = static_cast<char *>(workspace);
    a.counters = reinterpret_cast<int32_t *>(ws + L.counters);
    a.part = reinterpret_cast<float *>(ws + L.part);
    attn_schedule(a, true);
    FusedArgs f{};
    f.cu_new = cu_new;
    f.total_new = total_new;
    f.k_new = k_new;
    f.v_new = v_new;
    f.kc_new = kc_new;
    f.k_pool = cache->k_pool;
    f.v_pool = cache->v_pool;
    f.kc_pool = cache->kc_pool;
    f.q_idx = q_idx;
    f.w = w;
    f.num_idx_heads = num_idx_heads;
    f.k_per_seq = k_per_seq;
    f.sel = sel;
    f.cnt = cnt;
    f.hdr = reinterpret_cast<int32_t *>(ws + L.hdr);
    f.sel_count = reinterpret_cast<int32_t *>(ws + L.sel_count);
    f.flags = reinterpret_cast<int32_t *>(ws + L.flags);
    f.cand = reinterpret_cast<unsigned long long *>(ws + L.cand);
    return from_cuda(launch_decode_fused(a, f, reinterpret_cast<cudaStream_t>(stream)));
}

int dsa_sparse_attn_prefill(const dsa_kv_cache *cache, const dsa_seqs *seqs, const dsa_queries *queries,
                            const void *q, int32_t num_q_heads, const int32_t *sel, const int32_t *cnt,
                            int32_t k_max, float sm_scale, void *out, float *lse, int32_t *dev_err,
                            dsa_stream_t stream) {
    AttnArgs a;
    int rc = attn_common(cache, seqs, queries, q, num_q_heads, sel, cnt, k_max, sm_scale, out, lse, dev_err, a);
    if (rc) return rc;
    if (queries->total_q == 0) return DSA_OK;
    attn_schedule(a, false);   // whole pairs per CTA: no partial states, no workspace
    return from_cuda(launch_sparse_attn(a, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
