// extern "C" entry points of libmla_b200: host-side validation, workspace
// layout and kernel launches.  Every function is asynchronous on the caller's
// stream; nothing here allocates, synchronises or keeps pointers.
#include <math.h>
#include <stdint.h>

#include "mla_internal.cuh"

namespace {

using namespace mla;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int auto_splits(int B, int n_q, int H) {
    const int rowblocks = (n_q * H + 15) / 16;
    const int ctas = B * rowblocks;
    int s = (2 * 148 + ctas - 1) / ctas;
    return s < 1 ? 1 : (s > 64 ? 64 : s);
}

struct DecodeWs {
    size_t o_part, lse_part, total;
};

DecodeWs decode_ws_layout(int B, int n_q, int H, int S) {
    const size_t rows = static_cast<size_t>(B) * n_q * H;
    DecodeWs w;
    w.o_part = 0;
    w.lse_part = rows * S * kDc * sizeof(float);
    w.total = w.lse_part + ((rows * S * sizeof(float) + 255) / 256) * 256;
    return w;
}

mla_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

int max_pairs_per_group(int G) { return kMaxPairs / G > 1 ? kMaxPairs / G : 1; }

// Few query rows (n_q * H <= 32): the one-SM kernel (one row group, up to kMaxSmCtas CTAs) instead of CTA pairs.
bool one_sm_path(int n_q, int H) { return static_cast<int64_t>(n_q) * H <= kMaxSmRows; }

// ---- tensor-core path: segment partials [G][slots][rs rows] float2 (m, l), then (1024-aligned)
//      [G][slots] blocks of rs rows x 512 fp32 O, each stored as [128 column groups of 4][rs rows] x float4,
//      then (1024-aligned) the merged latent output o_lat as bf16 operand tiles, [H][olat_rows(T)] x 1 KB.
//      A slot per (sequence + CTA pair of the group): a pair's range starts at most one piece into a sequence.
struct TcWs {
    int G, slots, rs;  // rs: rows per slot (128; kMaxSmRows on the one-SM path)
    size_t ml_part, o_part, olat, total;
};

size_t align1k(size_t x) { return ((x + 1023) / 1024) * 1024; }

TcWs tc_ws_layout(int B, int n_q, int H) {
    TcWs w;
    w.G = (n_q * H + 127) / 128;
    // a group gets at most max(1, kMaxPairs / G) CTA pairs (long query chunks: many groups, few pairs each);
    // with few query rows the one-SM kernel's up to kMaxSmCtas CTAs share the single group
    w.slots = B + (one_sm_path(n_q, H) ? kMaxSmCtas : max_pairs_per_group(w.G));
    w.rs = one_sm_path(n_q, H) ? kMaxSmRows : 128;
    const size_t rows = static_cast<size_t>(w.G) * w.slots * w.rs;
    w.ml_part = 0;
    w.o_part = align1k(rows * sizeof(float2));
    w.olat = align1k(w.o_part + rows * kDc * sizeof(float));
    w.total = w.olat + static_cast<size_t>(H) * olat_rows(B * n_q) * 1024;
    return w;
}

// Work units (CTA pairs, or CTAs of the one-SM kernel) per row group; the attend and finish phases derive
// the same number, so the merge finds every piece.
int tc_clusters_per_group(int G, int num_splits, bool one_sm) {
    if (one_sm) {
        int n = decode_sm_ctas();
        if (n <= 0) return 0;
        if (num_splits > 0 && num_splits < n) n = num_splits;
        return n;
    }
    const int total = decode_tc_clusters();
    if (total <= 0) return 0;
    int pg = total / G;
    if (pg < 1) pg = 1;
    if (num_splits > 0 && num_splits < pg) pg = num_splits;
    return pg < max_pairs_per_group(G) ? pg : max_pairs_per_group(G);
}

constexpr int64_t kMaxPoolBlocks = 0x7FFFFFFF;                 // block-table entries are int32
constexpr int kMaxTableBlocks = 0x7FFFFFFF / kBlockTokens;      // positions are int32

mla_status check_decode_shape(int B, int64_t cap_blocks, int max_blocks, int n_q, int H, int num_splits) {
    if (B < 0 || cap_blocks < 0 || cap_blocks > kMaxPoolBlocks || max_blocks < 0 || max_blocks > kMaxTableBlocks)
        return MLA_ERR_INVALID_ARG;
    if (B > 0 && (cap_blocks < 1 || max_blocks < 1)) return MLA_ERR_INVALID_ARG;
    if (H < 1 || H > kMaxHeads || n_q < 1 || n_q > kMaxNq || num_splits < 0 || num_splits > 256)
        return MLA_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<int64_t>(B) * n_q > 0x7FFFFFFF / kMaxHeads) return MLA_ERR_UNSUPPORTED_SHAPE;
    return MLA_OK;
}

}  // namespace

extern "C" {

int mla_abi_version(void) { return 2; }

const char* mla_status_string(int status) {
    switch (status) {
        case MLA_OK: return "ok";
        case MLA_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, negative or too large size)";
        case MLA_ERR_UNSUPPORTED_SHAPE:
            return "unsupported shape (H in 1..128, n_q in 1..16, splits in 0..256, B * n_q * 128 < 2^31)";
        case MLA_ERR_CUDA: return "CUDA runtime error";
        case MLA_ERR_WORKSPACE: return "workspace too small";
        default: return "unknown status";
    }
}

const char* mla_device_status_string(int32_t w) {
    if (w == 0) return "ok";
    if (w & MLA_DEVERR_TIMEOUT) return "bounded wait expired in a pipelined kernel";
    if (w & MLA_DEVERR_ROW_RANGE) return "cache block outside [0, cap_blocks)";
    if (w & MLA_DEVERR_POS_RANGE) return "position outside the RoPE table";
    if (w & MLA_DEVERR_KV_LEN) return "kv_len smaller than n_q";
    return "unknown device error bits";
}

mla_status mla_rope_table_fill(float* table, int64_t rope_len, double base) {
    if (!table || rope_len < 0 || !(base > 0.0)) return MLA_ERR_INVALID_ARG;
    double theta[kDr / 2];
    for (int i = 0; i < kDr / 2; ++i) theta[i] = pow(base, -2.0 * i / (double)kDr);
    for (int64_t p = 0; p < rope_len; ++p) {
        for (int i = 0; i < kDr / 2; ++i) {
            const double ang = (double)p * theta[i];
            table[p * kDr + 2 * i] = (float)cos(ang);
            table[p * kDr + 2 * i + 1] = (float)sin(ang);
        }
    }
    return MLA_OK;
}

mla_status mla_absorb_q(const void* q_nope, const void* q_rope, const int32_t* pos, const void* W_UK,
                        const float* rope_table, int64_t rope_len, int T, int H, void* q_out,
                        int32_t* dev_status, mla_stream stream) {
    if (T < 0 || rope_len < 0) return MLA_ERR_INVALID_ARG;
    if (H < 1 || H > kMaxHeads) return MLA_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MLA_OK;
    if (!q_nope || !q_rope || !W_UK || !q_out || (pos && !rope_table)) return MLA_ERR_INVALID_ARG;
    if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(W_UK) || !aligned16(q_out)) return MLA_ERR_INVALID_ARG;
    return cuda_status(launch_absorb_tc(static_cast<const uint16_t*>(q_nope), static_cast<const uint16_t*>(q_rope),
                                       pos, static_cast<const uint16_t*>(W_UK), rope_table, rope_len, T, H,
                                       static_cast<uint16_t*>(q_out), dev_status,
                                       static_cast<cudaStream_t>(stream)));
}

mla_status mla_query_up(const void* c_q, const void* W_UQ, const void* W_QR, int T, int H, int d_cq,
                        void* q_nope, void* q_rope, int32_t* dev_status, mla_stream stream) {
    if (T < 0) return MLA_ERR_INVALID_ARG;
    if (H < 1 || H > kMaxHeads || d_cq < 64 || d_cq > 16384 || d_cq % 64 != 0) return MLA_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MLA_OK;
    if (!c_q || !W_UQ || !W_QR || !q_nope || !q_rope) return MLA_ERR_INVALID_ARG;
    if (!aligned16(c_q) || !aligned16(W_UQ) || !aligned16(W_QR) || !aligned16(q_nope) || !aligned16(q_rope))
        return MLA_ERR_INVALID_ARG;
    return cuda_status(launch_query_up(static_cast<const uint16_t*>(c_q), static_cast<const uint16_t*>(W_UQ),
                                       static_cast<const uint16_t*>(W_QR), T, H, d_cq, static_cast<uint16_t*>(q_nope),
                                       static_cast<uint16_t*>(q_rope), dev_status, static_cast<cudaStream_t>(stream)));
}

mla_status mla_query_absorb(const void* c_q, const void* W_UQ, const void* W_QR, const void* W_UK, const int32_t* pos,
                            const float* rope_table, int64_t rope_len, int T, int H, int d_cq, void* q_out,
                            int32_t* dev_status, mla_stream stream) {
    if (T < 0 || rope_len < 0) return MLA_ERR_INVALID_ARG;
    if (H < 1 || H > kMaxHeads || d_cq < 64 || d_cq > 16384 || d_cq % 64 != 0) return MLA_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MLA_OK;
    if (!c_q || !W_UQ || !W_QR || !W_UK || !q_out || (pos && !rope_table)) return MLA_ERR_INVALID_ARG;
    if (!aligned16(c_q) || !aligned16(W_UQ) || !aligned16(W_QR) || !aligned16(W_UK) || !aligned16(q_out))
        return MLA_ERR_INVALID_ARG;
    return cuda_status(launch_query_absorb(static_cast<const uint16_t*>(c_q), static_cast<const uint16_t*>(W_UQ),
                                           static_cast<const uint16_t*>(W_QR), static_cast<const uint16_t*>(W_UK), pos,
                                           rope_table, rope_len, T, H, d_cq, static_cast<uint16_t*>(q_out),
                                           dev_status, static_cast<cudaStream_t>(stream)));
}

mla_status mla_append_cache(void* cache, int64_t cap_blocks, const int32_t* block_table, int num_seqs,
                            int max_blocks, const int32_t* seq_idx, const int32_t* pos, const void* c_kv, const void* k_rope,
                            const float* rope_table, int64_t rope_len, int T, int32_t* dev_status,
                            mla_stream stream) {
    if (T < 0 || cap_blocks < 0 || cap_blocks > kMaxPoolBlocks || rope_len < 0 || max_blocks < 0 || num_seqs < 0)
        return MLA_ERR_INVALID_ARG;
    if (T == 0) return MLA_OK;
    if (!cache || !block_table || !seq_idx || !pos || !c_kv || !k_rope || !rope_table || max_blocks < 1 ||
        num_seqs < 1)
        return MLA_ERR_INVALID_ARG;
    if (!aligned16(cache) || !aligned16(c_kv) || !aligned16(k_rope) || !aligned16(rope_table))
        return MLA_ERR_INVALID_ARG;
    return cuda_status(launch_append_cache(static_cast<uint8_t*>(cache), cap_blocks, block_table, num_seqs,
                                           max_blocks, seq_idx, pos, static_cast<const uint16_t*>(c_kv),
                                           static_cast<const uint16_t*>(k_rope), rope_table, rope_len, T, dev_status,
                                           static_cast<cudaStream_t>(stream)));
}

size_t mla_decode_workspace_bytes(int B, int n_q, int H, int num_splits) {
    if (B < 0 || n_q < 1 || H < 1 || num_splits < 0) return 0;
    return tc_ws_layout(B, n_q, H).total;
}

mla_status mla_decode_attend(const void* q, const void* cache, int64_t cap_blocks, const int32_t* block_table,
                             int max_blocks, const int32_t* kv_len, int B, int n_q, int H, float scale,
                             int num_splits, void* workspace, size_t ws_bytes, int32_t* dev_status,
                             mla_stream stream) {
    mla_status st = check_decode_shape(B, cap_blocks, max_blocks, n_q, H, num_splits);
    if (st != MLA_OK) return st;
    if (!(scale > 0.f) || !isfinite(scale)) return MLA_ERR_INVALID_ARG;
    if (B == 0) return MLA_OK;
    if (!q || !cache || !block_table || !kv_len || !workspace) return MLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(cache) || !aligned16(workspace)) return MLA_ERR_INVALID_ARG;
    const TcWs lay = tc_ws_layout(B, n_q, H);
    if (ws_bytes < lay.total) return MLA_ERR_WORKSPACE;
    const bool one_sm = one_sm_path(n_q, H);
    const int pg = tc_clusters_per_group(lay.G, num_splits, one_sm);
    if (pg <= 0) return MLA_ERR_CUDA;
    char* ws = static_cast<char*>(workspace);
    if (one_sm)
        return cuda_status(launch_decode_sm(static_cast<const uint16_t*>(q), static_cast<const uint8_t*>(cache),
                                            cap_blocks, block_table, max_blocks, kv_len, B, n_q, H, scale, pg,
                                            reinterpret_cast<float*>(ws + lay.o_part),
                                            reinterpret_cast<float2*>(ws + lay.ml_part), lay.slots, lay.rs,
                                            dev_status, static_cast<cudaStream_t>(stream)));
    return cuda_status(launch_decode_tc(static_cast<const uint16_t*>(q), static_cast<const uint8_t*>(cache),
                                        cap_blocks, block_table, max_blocks, kv_len, B, n_q, H, scale, pg,
                                        reinterpret_cast<float*>(ws + lay.o_part),
                                        reinterpret_cast<float2*>(ws + lay.ml_part), lay.slots, dev_status,
                                        static_cast<cudaStream_t>(stream)));
}

mla_status mla_decode_finish(const int32_t* kv_len, int max_blocks, const void* W_UV, int B, int n_q, int H,
                             int num_splits, void* workspace, size_t ws_bytes, void* out, float* lse_out,
                             int32_t* dev_status, mla_stream stream) {
    mla_status st = check_decode_shape(B, B > 0 ? 1 : 0, max_blocks, n_q, H, num_splits);
    if (st != MLA_OK) return st;
    if (B == 0) return MLA_OK;
    if (!kv_len || !W_UV || !out || !workspace) return MLA_ERR_INVALID_ARG;
    if (!aligned16(W_UV) || !aligned16(out) || !aligned16(workspace)) return MLA_ERR_INVALID_ARG;
    const TcWs lay = tc_ws_layout(B, n_q, H);
    if (ws_bytes < lay.total) return MLA_ERR_WORKSPACE;
    const int pg = tc_clusters_per_group(lay.G, num_splits, one_sm_path(n_q, H));
    if (pg <= 0) return MLA_ERR_CUDA;
    char* ws = static_cast<char*>(workspace);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_merge(reinterpret_cast<const float*>(ws + lay.o_part),
                                 reinterpret_cast<const float2*>(ws + lay.ml_part), kv_len, max_blocks, B, n_q, H, pg,
                                 lay.slots, lay.rs, reinterpret_cast<uint8_t*>(ws + lay.olat), lse_out, dev_status,
                                 cs);
    if (e != cudaSuccess) return MLA_ERR_CUDA;
    return cuda_status(launch_upproj(reinterpret_cast<const uint8_t*>(ws + lay.olat),
                                     static_cast<const uint16_t*>(W_UV), B * n_q, H, static_cast<uint16_t*>(out),
                                     dev_status, cs));
}

mla_status mla_decode(const void* q, const void* cache, int64_t cap_blocks, const int32_t* block_table, int max_blocks,
                      const int32_t* kv_len, const void* W_UV, int B, int n_q, int H, float scale, int num_splits,
                      void* workspace, size_t ws_bytes, void* out, float* lse_out, int32_t* dev_status,
                      mla_stream stream) {
    if (B > 0 && (!W_UV || !out)) return MLA_ERR_INVALID_ARG;
    if (B > 0 && (!aligned16(W_UV) || !aligned16(out))) return MLA_ERR_INVALID_ARG;
    mla_status st = mla_decode_attend(q, cache, cap_blocks, block_table, max_blocks, kv_len, B, n_q, H, scale,
                                      num_splits, workspace, ws_bytes, dev_status, stream);
    if (st != MLA_OK || B == 0) return st;
    return mla_decode_finish(kv_len, max_blocks, W_UV, B, n_q, H, num_splits, workspace, ws_bytes, out, lse_out,
                             dev_status, stream);
}

size_t mla_decode_cudacore_workspace_bytes(int B, int n_q, int H, int num_splits) {
    if (B < 0 || n_q < 1 || H < 1 || num_splits < 0) return 0;
    const int S = num_splits ? num_splits : auto_splits(B, n_q, H);
    return decode_ws_layout(B, n_q, H, S).total;
}

mla_status mla_decode_cudacore(const void* q, const void* cache, int64_t cap_blocks, const int32_t* block_table,
                               int max_blocks, const int32_t* kv_len, const void* W_UV, int B, int n_q, int H,
                               float scale, int num_splits, void* workspace, size_t ws_bytes, void* out,
                               float* lse_out, int32_t* dev_status, mla_stream stream) {
    mla_status st = check_decode_shape(B, cap_blocks, max_blocks, n_q, H, num_splits);
    if (st != MLA_OK) return st;
    if (!(scale > 0.f) || !isfinite(scale)) return MLA_ERR_INVALID_ARG;
    if (B == 0) return MLA_OK;
    if (!q || !cache || !block_table || !kv_len || !W_UV || !out || !workspace) return MLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(cache) || !aligned16(W_UV) || !aligned16(out) || !aligned16(workspace))
        return MLA_ERR_INVALID_ARG;
    const int S = num_splits ? num_splits : auto_splits(B, n_q, H);
    const DecodeWs lay = decode_ws_layout(B, n_q, H, S);
    if (ws_bytes < lay.total) return MLA_ERR_WORKSPACE;
    float* o_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + lay.o_part);
    float* lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + lay.lse_part);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_decode_simt(static_cast<const uint16_t*>(q), static_cast<const uint8_t*>(cache),
                                       cap_blocks, block_table, max_blocks, kv_len, B, n_q, H, scale, S, o_part,
                                       lse_part, dev_status, cs);
    if (e != cudaSuccess) return MLA_ERR_CUDA;
    return cuda_status(launch_combine(o_part, lse_part, B * n_q, H, S, static_cast<const uint16_t*>(W_UV), out,
                                      lse_out, cs));
}

size_t mla_prefill_workspace_bytes(int L, int H) {
    if (L < 1 || H < 1) return 0;
    return 2 * prefill_rows_bytes(L, H);
}

mla_status mla_prefill_naive(const void* q_nope, const void* q_rope, const float* rope_table, int64_t rope_len,
                             const void* cache, int64_t cap_blocks, const int32_t* blocks, int L, int n,
                             const void* W_UK, const void* W_UV, int H, float scale, void* workspace,
                             size_t ws_bytes, void* out, float* lse_out, int32_t* dev_status, mla_stream stream) {
    if (n < 0 || L < 0 || cap_blocks < 0 || cap_blocks > kMaxPoolBlocks || rope_len < 0) return MLA_ERR_INVALID_ARG;
    if (H < 1 || H > kMaxHeads) return MLA_ERR_UNSUPPORTED_SHAPE;
    if (n == 0) return MLA_OK;
    if (n > L || L > rope_len || L >= (1 << 30) || cap_blocks < 1) return MLA_ERR_INVALID_ARG;
    if (static_cast<int64_t>(L) * H * kDh >= (int64_t(1) << 31)) return MLA_ERR_UNSUPPORTED_SHAPE;
    if (!(scale > 0.f) || !isfinite(scale)) return MLA_ERR_INVALID_ARG;
    if (!q_nope || !q_rope || !rope_table || !cache || !blocks || !W_UK || !W_UV || !workspace || !out)
        return MLA_ERR_INVALID_ARG;
    if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(rope_table) || !aligned16(cache) ||
        !aligned16(W_UK) || !aligned16(W_UV) || !aligned16(workspace) || !aligned16(out))
        return MLA_ERR_INVALID_ARG;
    const size_t rows = prefill_rows_bytes(L, H);
    if (ws_bytes < 2 * rows) return MLA_ERR_WORKSPACE;
    char* ws = static_cast<char*>(workspace);
    return cuda_status(launch_prefill_naive(
        static_cast<const uint16_t*>(q_nope), static_cast<const uint16_t*>(q_rope), rope_table,
        static_cast<const uint8_t*>(cache), cap_blocks, blocks, L, n, static_cast<const uint16_t*>(W_UK),
        static_cast<const uint16_t*>(W_UV), H, scale, reinterpret_cast<uint16_t*>(ws),
        reinterpret_cast<uint16_t*>(ws + rows), static_cast<uint16_t*>(out), lse_out, dev_status,
        static_cast<cudaStream_t>(stream)));
}

mla_status mla_splitkv_combine(const float* o_part, const float* lse_part, int T, int H, int num_splits,
                               const void* W_UV, void* out, float* lse_out, mla_stream stream) {
    if (T < 0) return MLA_ERR_INVALID_ARG;
    if (H < 1 || H > kMaxHeads || num_splits < 1 || num_splits > 256) return MLA_ERR_UNSUPPORTED_SHAPE;
    if (T == 0) return MLA_OK;
    if (!o_part || !lse_part || !out) return MLA_ERR_INVALID_ARG;
    if (!aligned16(o_part) || !aligned16(out) || (W_UV && !aligned16(W_UV))) return MLA_ERR_INVALID_ARG;
    return cuda_status(launch_combine(o_part, lse_part, T, H, num_splits, static_cast<const uint16_t*>(W_UV), out,
                                      lse_out, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
