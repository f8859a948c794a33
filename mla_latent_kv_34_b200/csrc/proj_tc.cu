// The per-head projections around the attend kernel, and the merge of its pieces.
//
//  absorb:  q_abs[t, h, :] = (W^UK_h)^T q_nope[t, h, :]          (512 = 128 x 512^T)
//           W^UK is folded into the query so scores are taken against the cached
//           latent ("两张账" page, "第一张账"; MLA explainer 2.2.1.1).  q^R is rotated at
//           the query position in fp32 exactly as the cache append rotates k^R
//           (explainer 2.2.2).
//  merge:   o_lat[t, h, :] = log-sum-exp merge of the attend kernel's pieces of one
//           sequence (each piece: unnormalised O over its key range, its running max
//           and sum), normalised and rounded to bf16.
//  upproj:  out[t, h, :] = W^UV_h o_lat[t, h, :]                   (128 = 128 x 512)
//           W^UV is applied after the aggregation in latent space ("两张账" page).
//
// absorb: one CTA per (128 latent columns, head, up to 128 query rows), so 4 CTAs share a
// head and each moves a quarter of W^UK_h; the weight quarter lands as two TMA boxes
// ([128 x 64] chunks, 128-byte swizzle) and is the MN-major A operand (M = latent
// column, K = head dim) of 8 MMAs against the staged q_nope rows (N = rows).  The result
// rows are staged in shared memory and leave as 16-byte stores.  (One CTA per head with all
// four quarters measured slower: 15.1 against 13.6 us at T = 32, 68.9 against 35.9 us at
// T = 256, ncu.)
// merge: one CTA per (column slice, sequence, row group); the launch picks the threads per row
// that share the sequence's pieces (1 to 16) and the slice width (8, 16 or 32 columns) from the
// expected pieces per sequence and the grid size.  The attend kernel writes the pieces in
// [column group][row] order; the merge writes o_lat into per-(head, 256-row block) tiles already
// in the swizzled K-major operand layout, so each K step of the up-projection takes its operand
// with one bulk copy.
// upproj: one CTA per (head, up to 256 rows), the contraction over the latent columns streamed
// through a ring of stages; W^UV_h's first chunks (all eight when T <= 64) are requested before
// the CTA waits for the merge, so the weight load overlaps it.  The bf16 result is staged in
// shared memory and whole output rows leave with 16-byte stores.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "mla_internal.cuh"
#include "sm100.cuh"

namespace mla {
using namespace sm100;

namespace proj {

constexpr int kWChunkBytes = 128 * 64 * 2;   // [128 rows x 64 columns] bf16 = 16 KB
constexpr int kTokBlock = 128;               // absorb: query rows per CTA (MMA N <= 128)
constexpr uint64_t kLimitNs = 2000000000ull;

// 16-byte unit u (0..7) of row r in a 128-byte swizzled row of a [rows x 64] chunk
__device__ __forceinline__ uint32_t swz(int r, int u) { return static_cast<uint32_t>(r * 128 + ((u ^ (r & 7)) << 4)); }

// ------------------------------------------------------------------ absorb

constexpr int kAbsThreads = 128;
constexpr int kAbsOffW = 0;                              // two weight chunks, 32 KB
constexpr int kAbsOffB = 2 * kWChunkBytes;               // q_nope rows: two [NT x 64] chunks, <= 32 KB
constexpr int kAbsOffPos = kAbsOffB + kTokBlock * 128 * 2;  // query positions of the rows (RoPE CTAs)
constexpr int kAbsOffBar = kAbsOffPos + kTokBlock * 4;
constexpr int kAbsSmemBytes = kAbsOffBar + 64;

__global__ void __launch_bounds__(kAbsThreads) absorb_tc_kernel(
    const __grid_constant__ CUtensorMap wuk_map, const uint16_t* __restrict__ q_nope,
    const uint16_t* __restrict__ q_rope, const int32_t* __restrict__ pos, const float* __restrict__ rope_table,
    int64_t rope_len, int T, int H, uint16_t* __restrict__ q_out, int32_t* dev_status) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kAbsOffBar);  // 0: weights, 1: MMA done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kAbsOffBar + 16);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int mb = blockIdx.x;  // latent columns 128 mb .. 128 mb + 127
    const int h = blockIdx.y;
    const int t0 = blockIdx.z * kTokBlock;
    const int nt = min(kTokBlock, T - t0);
    const int NT = (nt + 15) & ~15;  // MMA N (multiple of 16)
    volatile int never = 0;
    if ((sbase & 1023u) != 0) {
        if (tid == 0) report(dev_status, MLA_DEVERR_TIMEOUT);
        return;
    }
    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
        prefetch_tmap(&wuk_map);
    }
    if (warp == 0) tmem_alloc(tmem_slot, kTokBlock);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    int32_t* pos_s = reinterpret_cast<int32_t*>(smem + kAbsOffPos);
    grid_dependency_wait();  // inputs may come from the previous kernel on the stream
    // query positions of the RoPE CTAs' rows (-1: none given; -2: outside the table, reported, and that
    // row's RoPE part is left unwritten)
    if (mb == 0 && tid < nt) {
        int32_t pp = -1;
        if (pos) {
            pp = pos[t0 + tid];
            if (pp < 0 || pp >= rope_len) {
                report(dev_status, MLA_DEVERR_POS_RANGE);
                pp = -2;
            }
        }
        pos_s[tid] = pp;
    }
    if (tid == 0) {
        mbar_arrive_expect_tx(&bars[0], 2 * kWChunkBytes);
        tma_load_3d(sbase + kAbsOffW, &wuk_map, 0, h * 128, 2 * mb, &bars[0]);
        tma_load_3d(sbase + kAbsOffW + kWChunkBytes, &wuk_map, 0, h * 128, 2 * mb + 1, &bars[0]);
    }
    // B operand: q_nope rows t (N) x 128 (K), two swizzled [NT x 64] chunks; rows >= nt are zero.  Eight
    // 16-byte loads per thread in flight at a time.
    for (int base = 0; base < NT * 16; base += 8 * kAbsThreads) {
        uint4 v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int idx = base + tid + k * kAbsThreads, r = idx >> 4, u16 = idx & 15;  // 16 units per row
            v[k] = make_uint4(0, 0, 0, 0);
            if (r < nt) v[k] = reinterpret_cast<const uint4*>(q_nope + (static_cast<int64_t>(t0 + r) * H + h) * kDh)[u16];
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int idx = base + tid + k * kAbsThreads, r = idx >> 4, u16 = idx & 15;
            if (r < NT) *reinterpret_cast<uint4*>(smem + kAbsOffB + (u16 >> 3) * NT * 128 + swz(r, u16 & 7)) = v[k];
        }
    }
    fence_proxy_async_cta();
    __syncthreads();
    bool ok = true;
    if (tid == 0) {
        ok = mbar_wait(&bars[0], 0, &never, kLimitNs);
        if (ok) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(128, NT, true, false);
            // A = W^UK_h^T (M = latent c, K = i): MN-major; the 128 columns span the two chunks
            const uint64_t a0 = sdesc_sw128(sbase + kAbsOffW, kWChunkBytes, 1024);
            const uint64_t b0 = sdesc_sw128(sbase + kAbsOffB, 16, 1024);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint64_t ad = a0 + static_cast<uint64_t>((k * 2048) >> 4);
                const uint64_t bd = b0 + static_cast<uint64_t>(((k >> 2) * NT * 128 + (k & 3) * 32) >> 4);
                mma_ss(tmem, ad, bd, idesc, k > 0 ? 1u : 0u);
            }
            mma_commit(smem_u32(&bars[1]));
        } else {
            report(dev_status, MLA_DEVERR_TIMEOUT);
        }
    }
    grid_dependents_launch();
    // RoPE part on CUDA cores meanwhile (the first CTA of each head and row block does it), the same
    // arithmetic as the cache append.  A thread takes 16-byte units (row j, dims 8u .. 8u + 7 = pairs
    // 4u .. 4u + 3) four at a time, with every load of a batch in flight together; the positions were
    // staged before the first barrier above.
    if (mb == 0) {
        for (int base = 0; base < nt * 8; base += 4 * kAbsThreads) {
            uint4 x[4];
            float4 cs[4][2];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int idx = base + tid + k * kAbsThreads, j = idx >> 3, u = idx & 7;
                x[k] = make_uint4(0, 0, 0, 0);
                cs[k][0] = cs[k][1] = make_float4(1.f, 0.f, 1.f, 0.f);
                if (j < nt) {
                    x[k] = reinterpret_cast<const uint4*>(q_rope + (static_cast<int64_t>(t0 + j) * H + h) * kDr)[u];
                    const int32_t pp = pos_s[j];
                    if (pp >= 0) {
                        const float4* row = reinterpret_cast<const float4*>(rope_table + static_cast<int64_t>(pp) * kDr);
                        cs[k][0] = row[2 * u];
                        cs[k][1] = row[2 * u + 1];
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int idx = base + tid + k * kAbsThreads, j = idx >> 3, u = idx & 7;
                if (j >= nt || pos_s[j] == -2) continue;
                uint4 y = x[k];
                if (pos_s[j] >= 0) {
                    const uint32_t w[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
                    const float c[8] = {cs[k][0].x, cs[k][0].y, cs[k][0].z, cs[k][0].w,
                                        cs[k][1].x, cs[k][1].y, cs[k][1].z, cs[k][1].w};
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {  // pair 4u + e: (cos, sin) = (c[2e], c[2e + 1])
                        const float x0 = bf16_to_f32(static_cast<uint16_t>(w[e] & 0xFFFFu));
                        const float x1 = bf16_to_f32(static_cast<uint16_t>(w[e] >> 16));
                        o[e] = pack_bf16x2(__fsub_rn(__fmul_rn(x0, c[2 * e]), __fmul_rn(x1, c[2 * e + 1])),
                                           __fadd_rn(__fmul_rn(x0, c[2 * e + 1]), __fmul_rn(x1, c[2 * e])));
                    }
                    y = make_uint4(o[0], o[1], o[2], o[3]);
                }
                reinterpret_cast<uint4*>(q_out + (static_cast<int64_t>(t0 + j) * H + h) * kRow + kDc)[u] = y;
            }
        }
    }
    ok = __syncthreads_and(ok);
    bool done = false;
    if (ok) {
        // D: lane = latent column 128 mb + 32 warp + lane, column = row t.  Once the MMAs are done the B
        // operand's space is free: row j of the result goes there as 256 bytes of bf16, so that it leaves
        // as 16-byte stores (a thread per column would store 2 bytes into each of 32 rows).
        done = mbar_wait(&bars[1], 0, &never, kLimitNs);
        __syncwarp();
        tc_fence_after();
        done = __all_sync(0xffffffffu, done);
        if (done) {
            uint16_t* stage = reinterpret_cast<uint16_t*>(smem + kAbsOffB);
            const int cl = 32 * warp + lane;
            for (int j0 = 0; j0 < NT; j0 += 32) {
                uint32_t v[32];
                const uint32_t ta = tmem + (static_cast<uint32_t>(32 * warp) << 16) + j0;
                if (NT - j0 >= 32) tmem_ld32(ta, v);
                else tmem_ld16(ta, v);  // NT is a multiple of 16
                tmem_wait_ld();
                const int jn = min(32, nt - j0);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j < jn) stage[(j0 + j) * 128 + cl] = f32_to_bf16_rne(__uint_as_float(v[j]));
            }
        } else if (lane == 0) {
            report(dev_status, MLA_DEVERR_TIMEOUT);
        }
    }
    if (__syncthreads_and(done)) {
        // rows t0 .. t0 + nt - 1, latent columns 128 mb .. 128 mb + 127: 16 units of 16 bytes per row
        for (int idx = tid; idx < nt * 16; idx += kAbsThreads) {
            const int j = idx >> 4, u = idx & 15;
            const uint4 y = *reinterpret_cast<const uint4*>(smem + kAbsOffB + j * 256 + u * 16);
            reinterpret_cast<uint4*>(q_out + (static_cast<int64_t>(t0 + j) * H + h) * kRow + 128 * mb)[u] = y;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTokBlock);
    }
}

// ------------------------------------------------------------------ merge

// Byte offset of row t of head h, latent unit (chunk c, unit u) in the o_lat tiles: per head, the rows
// are cut into blocks of kOlatBlock (the last one olat_rows(T) - kOlatBlock * (blocks - 1) rows); a block
// is eight [rows x 64] chunks, each 128-byte swizzled, so chunk c of a block is the K-major B operand of
// the up-projection's K step c and arrives with one bulk copy.
constexpr int kOlatBlock = 256;
__device__ __forceinline__ int64_t olat_offset(int T, int h, int t, int c, int u) {
    const int Tp = olat_rows(T);
    const int tb = t / kOlatBlock, i = t % kOlatBlock;
    const int rows = min(kOlatBlock, Tp - kOlatBlock * tb);
    return (static_cast<int64_t>(h) * Tp + kOlatBlock * tb) * 1024 + c * rows * 128 + swz(i, u);
}

// One CTA per (column slice, sequence, row group); blockDim = rows x kSplit with rows = min(128, rows per slot).
// Row r of the group is merged by kSplit threads (neighbouring lanes), each over every kSplit-th piece of the
// sequence with its own running maximum; their partial results are combined with warp shuffles.  A thread
// covers kVec column groups of 4 (slice = 4 kVec columns, 128 / kVec slices per row) and issues the loads of
// 8 / kVec pieces before it uses any, so that every thread has eight 16-byte loads in flight per round trip.
// The launch picks kSplit from the expected pieces per sequence and kVec from the number of CTAs, so that a
// few long sequences cut into many pieces still spread over the whole GPU.  A thread's loads of one piece
// are kVec 16-byte column groups of its row (the attend kernel's [column group][row] order).
template <int kSplit, int kVec>
__global__ void __launch_bounds__(512) merge_kernel(
    const float* __restrict__ o_part, const float2* __restrict__ ml_part, const int32_t* __restrict__ kv_len,
    int max_blocks, int B, int n_q, int H, int P_g, int slots, int rs, uint8_t* __restrict__ olat,
    float* __restrict__ lse_out) {
    static_assert(kSplit >= 1 && kSplit <= 32 && (kSplit & (kSplit - 1)) == 0, "kSplit: power of two <= 32");
    static_assert(kVec == 2 || kVec == 4 || kVec == 8, "kVec: 2, 4 or 8 column groups");
    constexpr int kBatch = 8 / kVec;  // pieces whose loads are in flight together
    __shared__ int red[2][16];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nthr = blockDim.x, nwarps = nthr >> 5;
    const int slice = blockIdx.x, b = blockIdx.y, g = blockIdx.z;
    const int r = tid / kSplit, k = tid % kSplit;
    // tiles of all sequences (the attend kernel's range split depends on the total) and before b.  The
    // lengths are an input of the decode call, the same for both phases, so they are read before the wait
    // for the attend kernel's pieces and this part overlaps its tail.
    int s_all = 0, s_pre = 0;
    for (int i = tid; i < B; i += nthr) {
        const int n = valid_seq_tiles(kv_len[i], n_q, max_blocks);
        s_all += n;
        if (i < b) s_pre += n;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        s_all += __shfl_xor_sync(0xffffffffu, s_all, o);
        s_pre += __shfl_xor_sync(0xffffffffu, s_pre, o);
    }
    if (lane == 0) {
        red[0][warp] = s_all;
        red[1][warp] = s_pre;
    }
    __syncthreads();
    int Nt = 0, ts = 0;
    for (int w = 0; w < nwarps; ++w) {
        Nt += red[0][w];
        ts += red[1][w];
    }
    const int ntb = valid_seq_tiles(kv_len[b], n_q, max_blocks);
    grid_dependency_wait();  // the pieces come from the attend kernel
    grid_dependents_launch();
    const int R = n_q * H;
    const int rr = g * 128 + r;
    const bool row_ok = r < rs && rr < R;  // (no early exit: the shuffles below need every lane)
    // pieces of sequence b: the attend kernel's pairs whose tile range [lo, hi) meets [ts, ts + ntb)
    int p_first = 0, p_last = -1;
    if (ntb > 0 && Nt > 0 && row_ok) {
        p_first = static_cast<int>((static_cast<int64_t>(ts + 1) * P_g - 1) / Nt);
        p_last = static_cast<int>((static_cast<int64_t>(ts + ntb) * P_g - 1) / Nt);
    }
    const int64_t seg0 = static_cast<int64_t>(g) * slots + b;  // slot of piece p: seg0 + p
    // with more pairs than tiles some pairs in [p_first, p_last] have empty ranges and wrote nothing
    auto live = [&](int p) {
        const int lo = static_cast<int>((static_cast<int64_t>(p) * Nt) / P_g);
        const int hi = static_cast<int>((static_cast<int64_t>(p + 1) * Nt) / P_g);
        return max(lo, ts) < min(hi, ts + ntb);
    };
    float M = -CUDART_INF_F, z = 0.f;
    float acc[4 * kVec];
#pragma unroll
    for (int i = 0; i < 4 * kVec; ++i) acc[i] = 0.f;
    const int cg0 = kVec * slice;  // column groups cg0 .. cg0 + kVec - 1 = columns 4 cg0 .. 4 cg0 + 4 kVec - 1
    for (int p0 = p_first + k; p0 <= p_last; p0 += kSplit * kBatch) {
        // segment partials: [column group of 4][rs rows] x float4; every load of the batch goes out before
        // the (m, l) tests
        float4 v[kBatch][kVec];
        float2 ml[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int p = p0 + u * kSplit;
            ml[u] = make_float2(-CUDART_INF_F, 0.f);
            if (p <= p_last && live(p)) {
                const float4* src = reinterpret_cast<const float4*>(o_part) + ((seg0 + p) * 128 + cg0) * rs + r;
#pragma unroll
                for (int i = 0; i < kVec; ++i) v[u][i] = src[i * rs];
                ml[u] = ml_part[(seg0 + p) * rs + r];
            }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (ml[u].x == -CUDART_INF_F) continue;
            const float Mn = fmaxf(M, ml[u].x);
            const float sc = exp2f(M - Mn), w = exp2f(ml[u].x - Mn);
            z = z * sc + ml[u].y * w;
            M = Mn;
#pragma unroll
            for (int i = 0; i < kVec; ++i) {
                acc[4 * i] = fmaf(w, v[u][i].x, acc[4 * i] * sc);
                acc[4 * i + 1] = fmaf(w, v[u][i].y, acc[4 * i + 1] * sc);
                acc[4 * i + 2] = fmaf(w, v[u][i].z, acc[4 * i + 2] * sc);
                acc[4 * i + 3] = fmaf(w, v[u][i].w, acc[4 * i + 3] * sc);
            }
        }
    }
    // combine the row's kSplit partial merges (neighbouring lanes)
    float Mr = M;
#pragma unroll
    for (int o = 1; o < kSplit; o <<= 1) Mr = fmaxf(Mr, __shfl_xor_sync(0xffffffffu, Mr, o));
    const float sc = (M == -CUDART_INF_F) ? 0.f : exp2f(M - Mr);
    z *= sc;
#pragma unroll
    for (int o = 1; o < kSplit; o <<= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
#pragma unroll
    for (int i = 0; i < 4 * kVec; ++i) {
        float a = acc[i] * sc;
#pragma unroll
        for (int o = 1; o < kSplit; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        acc[i] = a;
    }
    if (!row_ok) return;
    const int j = rr / H, h = rr % H;
    const int t = b * n_q + j;
    const int T = B * n_q;
    const float inv = (z > 0.f) ? 1.f / z : 0.f;
    // the slice's kVec / 2 units of 8 columns (16 bytes of bf16); thread k writes the units q with
    // q % kSplit == k.  Column 4 cg0 + 8 q is in chunk (4 cg0 + 8 q) / 64, unit ((4 cg0 + 8 q) % 64) / 8.
#pragma unroll
    for (int q = 0; q < kVec / 2; ++q) {
        if (q % kSplit != k) continue;
        const int col = 4 * cg0 + 8 * q;
        uint4 y;
        y.x = pack_bf16x2(acc[8 * q] * inv, acc[8 * q + 1] * inv);
        y.y = pack_bf16x2(acc[8 * q + 2] * inv, acc[8 * q + 3] * inv);
        y.z = pack_bf16x2(acc[8 * q + 4] * inv, acc[8 * q + 5] * inv);
        y.w = pack_bf16x2(acc[8 * q + 6] * inv, acc[8 * q + 7] * inv);
        *reinterpret_cast<uint4*>(olat + olat_offset(T, h, t, col >> 6, (col & 63) >> 3)) = y;
    }
    if (slice == 0 && k == 0 && lse_out)
        lse_out[static_cast<int64_t>(t) * H + h] = (z > 0.f) ? (Mr + log2f(z)) * 0.69314718055994530942f : -CUDART_INF_F;
}

// ------------------------------------------------------------------ up-projection

constexpr int kUpThreads = 128;

// Shared-memory plan of the up-projection: kStages stages of [W^UV chunk (16 KB) | o_lat chunk (kRows x 128 B)],
// then the barriers (full[kStages], empty[kStages], done) and the TMEM address.
template <int kRows, int kStages>
struct UpPlan {
    static constexpr int kOffB = kWChunkBytes;
    static constexpr int kStageBytes = kWChunkBytes + kRows * 128;
    static constexpr int kOffBar = kStages * kStageBytes;
    static constexpr int kSmemBytes = kOffBar + 256;
    static_assert(kStageBytes % 1024 == 0 && kRows * kDh * 2 <= kOffBar, "stages 1024-aligned; output staging fits");
    static_assert(8 * (2 * kStages + 1) + 4 <= 256 && kSmemBytes <= 227 * 1024, "barriers and stages fit");
};

// One CTA per (head, block of up to kRows o_lat rows).  The contraction over the 512 latent columns streams
// through a ring of kStages stages, one 64-column chunk per stage: W^UV_h's chunk as a [128 x 64] TMA box (the
// K-major A operand, M = output dim) and the o_lat block's chunk as one bulk copy (the K-major B operand,
// N = rows).  W^UV is an input of the decode call, never written by the kernels before this one in it, so
// its first boxes are requested before the CTA waits for the merge.  With at most 64 rows (kRows = 64) the
// eight stages hold the whole of W^UV_h, which is then all requested before the wait, and the o_lat chunks
// all leave together after it.  The result is staged in shared memory as bf16 rows and leaves as 16-byte
// stores (each output row is 256 contiguous bytes).
template <int kRows, int kStages>
__global__ void __launch_bounds__(kUpThreads) upproj_kernel(const __grid_constant__ CUtensorMap wuv_map,
                                                           const uint8_t* __restrict__ olat, int T, int H,
                                                           uint16_t* __restrict__ out, int32_t* dev_status) {
    using Plan = UpPlan<kRows, kStages>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Plan::kOffBar);  // full[kStages], empty[kStages], done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Plan::kOffBar + 8 * (2 * kStages + 1));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x;
    const int t0 = blockIdx.y * kRows;
    const int nt = min(kRows, T - t0);
    const int Tp = olat_rows(T);
    const int NT = min(kRows, Tp - t0);  // rows of this o_lat block (a multiple of 16)
    const uint32_t chunk_bytes = static_cast<uint32_t>(NT) * 128u;
    const uint8_t* blk = olat + (static_cast<int64_t>(h) * Tp + t0) * 1024;  // chunk c at c * NT * 128
    volatile int never = 0;
    if ((sbase & 1023u) != 0) {
        if (tid == 0) report(dev_status, MLA_DEVERR_TIMEOUT);
        return;
    }
    if (tid == 0) {
        for (int i = 0; i < 2 * kStages + 1; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        prefetch_tmap(&wuv_map);
        for (int c = 0; c < kStages; ++c) {
            mbar_arrive_expect_tx(&bars[c], kWChunkBytes + chunk_bytes);
            tma_load_3d(sbase + c * Plan::kStageBytes, &wuv_map, 0, h * 128, c, &bars[c]);
        }
    }
    if (warp == 0) tmem_alloc(tmem_slot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    grid_dependency_wait();  // o_lat comes from the merge kernel
    bool ok = true;
    if (warp == 0 && lane == 0) {
        // producer: the o_lat halves of the first kStages stages, then both halves of the remaining chunks (if
        // any) as stages free
        const uint64_t once = l2_policy_evict_first();
        for (int c = 0; c < kStages; ++c)
            bulk_load_hint(sbase + c * Plan::kStageBytes + Plan::kOffB, blk + c * chunk_bytes, chunk_bytes, &bars[c], once);
        for (int c = kStages; ok && c < 8; ++c) {
            const int s = c % kStages;
            ok = mbar_wait(&bars[kStages + s], 0, &never, kLimitNs);
            if (!ok) break;
            mbar_arrive_expect_tx(&bars[s], kWChunkBytes + chunk_bytes);
            tma_load_3d(sbase + s * Plan::kStageBytes, &wuv_map, 0, h * 128, c, &bars[s]);
            bulk_load_hint(sbase + s * Plan::kStageBytes + Plan::kOffB, blk + c * chunk_bytes, chunk_bytes, &bars[s], once);
        }
        if (!ok) report(dev_status, MLA_DEVERR_TIMEOUT);
    } else if (warp == 1 && lane == 0) {
        // MMA issuer: out^T[d, t] += W^UV_h[d, chunk] o_lat[t, chunk], four K = 16 steps per chunk
        const uint32_t idesc = idesc_bf16_f32(128, NT, false, false);
        for (int c = 0; ok && c < 8; ++c) {
            const int s = c % kStages;
            ok = mbar_wait(&bars[s], static_cast<uint32_t>(c / kStages), &never, kLimitNs);
            if (!ok) break;
            tc_fence_after();
            const uint64_t a0 = sdesc_sw128(sbase + s * Plan::kStageBytes, 16, 1024);
            const uint64_t b0 = sdesc_sw128(sbase + s * Plan::kStageBytes + Plan::kOffB, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ss(tmem, a0 + static_cast<uint64_t>((kk * 32) >> 4), b0 + static_cast<uint64_t>((kk * 32) >> 4),
                       idesc, (c > 0 || kk > 0) ? 1u : 0u);
            mma_commit(smem_u32(&bars[kStages + s]));  // stage s free once these MMAs are done
        }
        if (!ok) report(dev_status, MLA_DEVERR_TIMEOUT);
        mma_commit(smem_u32(&bars[2 * kStages]));  // also after a failure: TMEM is freed only once it fires
    }
    ok = __syncthreads_and(ok);
    {
        const bool done = mbar_wait(&bars[2 * kStages], 0, &never, kLimitNs);
        __syncwarp();
        tc_fence_after();
        ok = __all_sync(0xffffffffu, done) && ok;
        if (ok) {
            // D: lane d = output dim of W^UV_h, column j = row t0 + j.  Every MMA is done, so the stages are
            // free: row j of the result goes to [j * 256, j * 256 + 256) as bf16
            const int d = 32 * warp + lane;
            for (int j0 = 0; j0 < NT; j0 += 32) {
                uint32_t v[32];
                const uint32_t ta = tmem + (static_cast<uint32_t>(32 * warp) << 16) + j0;
                if (NT - j0 >= 32) tmem_ld32(ta, v);
                else tmem_ld16(ta, v);  // NT is a multiple of 16
                tmem_wait_ld();
                const int jn = min(32, nt - j0);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j < jn)
                        *reinterpret_cast<uint16_t*>(smem + (j0 + j) * (kDh * 2) + 2 * d) =
                            f32_to_bf16_rne(__uint_as_float(v[j]));
            }
        } else if (lane == 0 && !done) {
            report(dev_status, MLA_DEVERR_TIMEOUT);
        }
    }
    ok = __syncthreads_and(ok);
    if (ok) {
        for (int i = tid; i < nt * (kDh * 2 / 16); i += kUpThreads) {
            const int j = i / (kDh * 2 / 16), q = i % (kDh * 2 / 16);
            reinterpret_cast<uint4*>(out + (static_cast<int64_t>(t0 + j) * H + h) * kDh)[q] =
                *reinterpret_cast<const uint4*>(smem + j * (kDh * 2) + 16 * q);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// W [H, 128, 512] bf16 viewed as (column within a 64-column chunk, row, chunk); one box = one chunk of a head.
bool weight_map(CUtensorMap* map, const uint16_t* W, int H) {
    auto encode = encode_fn();
    if (!encode) return false;
    cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(H) * 128, 8};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDc) * 2, 128};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(W), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch with programmatic stream serialization: the kernel may start while the previous kernel on the
// stream is finishing, and waits for it (grid_dependency_wait) before reading anything it could produce.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, int threads, int smem, cudaStream_t stream,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace proj

cudaError_t launch_absorb_tc(const uint16_t* q_nope, const uint16_t* q_rope, const int32_t* pos, const uint16_t* W_UK,
                             const float* rope_table, int64_t rope_len, int T, int H, uint16_t* q_out,
                             int32_t* dev_status, cudaStream_t stream) {
    CUtensorMap map;
    if (!proj::weight_map(&map, W_UK, H)) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(proj::absorb_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         proj::kAbsSmemBytes);
    if (e != cudaSuccess) return e;
    const dim3 grid(4, H, (T + proj::kTokBlock - 1) / proj::kTokBlock);
    return proj::launch_pdl(proj::absorb_tc_kernel, grid, proj::kAbsThreads, proj::kAbsSmemBytes, stream, map, q_nope,
                            q_rope, pos, rope_table, rope_len, T, H, q_out, dev_status);
}

namespace proj {

template <int kSplit, int kVec>
cudaError_t launch_merge_t(int rows, dim3 grid, cudaStream_t stream, const float* o_part, const float2* ml_part,
                           const int32_t* kv_len, int max_blocks, int B, int n_q, int H, int P_g, int slots, int rs,
                           uint8_t* olat, float* lse_out) {
    grid.x = 128 / kVec;
    return launch_pdl(merge_kernel<kSplit, kVec>, grid, rows * kSplit, 0, stream, o_part, ml_part, kv_len,
                      max_blocks, B, n_q, H, P_g, slots, rs, olat, lse_out);
}

template <int kSplit>
cudaError_t launch_merge_s(int vec, int rows, dim3 grid, cudaStream_t stream, const float* o_part,
                           const float2* ml_part, const int32_t* kv_len, int max_blocks, int B, int n_q, int H,
                           int P_g, int slots, int rs, uint8_t* olat, float* lse_out) {
    if (vec == 8)
        return launch_merge_t<kSplit, 8>(rows, grid, stream, o_part, ml_part, kv_len, max_blocks, B, n_q, H, P_g,
                                         slots, rs, olat, lse_out);
    if (vec == 4)
        return launch_merge_t<kSplit, 4>(rows, grid, stream, o_part, ml_part, kv_len, max_blocks, B, n_q, H, P_g,
                                         slots, rs, olat, lse_out);
    return launch_merge_t<kSplit, 2>(rows, grid, stream, o_part, ml_part, kv_len, max_blocks, B, n_q, H, P_g, slots,
                                     rs, olat, lse_out);
}

}  // namespace proj

cudaError_t launch_merge(const float* o_part, const float2* ml_part, const int32_t* kv_len, int max_blocks, int B,
                         int n_q, int H, int P_g, int slots, int rs, uint8_t* olat, float* lse_out,
                         int32_t* dev_status, cudaStream_t stream) {
    (void)dev_status;
    if (B < 1 || rs < 1 || rs > 128 || (rs & 31) != 0) return cudaErrorInvalidValue;
    const int G = (n_q * H + 127) / 128;
    const int rows = rs;  // rows per slot: 128, or 32 for the one-SM kernel's pieces
    // Threads per row: enough that none merges more than about five pieces (a sequence has about 1 + P_g / B
    // of them); then slices as wide as possible while the grid still has 64 K threads.  Measured at V2, 128K
    // and V2-Lite shapes (in a step, after the attend kernel), wider or narrower choices were slower: more
    // threads per row mostly add CTAs that wait, and narrow slices multiply the sequence-length prologue.
    int split = 1;
    while (split < 16 && rows * split * 2 <= 512 && static_cast<int64_t>(B) + P_g > int64_t(5) * split * B) split *= 2;
    int vec = 8;
    while (vec > 2 && int64_t(128 / vec) * B * G * rows * split < 65536) vec /= 2;
    const dim3 grid(1, B, G);
    switch (split) {
        case 1: return proj::launch_merge_s<1>(vec, rows, grid, stream, o_part, ml_part, kv_len, max_blocks, B, n_q,
                                               H, P_g, slots, rs, olat, lse_out);
        case 2: return proj::launch_merge_s<2>(vec, rows, grid, stream, o_part, ml_part, kv_len, max_blocks, B, n_q,
                                               H, P_g, slots, rs, olat, lse_out);
        case 4: return proj::launch_merge_s<4>(vec, rows, grid, stream, o_part, ml_part, kv_len, max_blocks, B, n_q,
                                               H, P_g, slots, rs, olat, lse_out);
        case 8: return proj::launch_merge_s<8>(vec, rows, grid, stream, o_part, ml_part, kv_len, max_blocks, B, n_q,
                                               H, P_g, slots, rs, olat, lse_out);
        default: return proj::launch_merge_s<16>(vec, rows, grid, stream, o_part, ml_part, kv_len, max_blocks, B,
                                                 n_q, H, P_g, slots, rs, olat, lse_out);
    }
}

cudaError_t launch_upproj(const uint8_t* olat, const uint16_t* W_UV, int T, int H, uint16_t* out, int32_t* dev_status,
                          cudaStream_t stream) {
    CUtensorMap map;
    if (!proj::weight_map(&map, W_UV, H)) return cudaErrorNotSupported;
    if (T <= 64) {  // one block per head, the whole W^UV_h resident
        using P = proj::UpPlan<64, 8>;
        cudaError_t e = cudaFuncSetAttribute(proj::upproj_kernel<64, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             P::kSmemBytes);
        if (e != cudaSuccess) return e;
        return proj::launch_pdl(proj::upproj_kernel<64, 8>, dim3(H, 1), proj::kUpThreads, P::kSmemBytes, stream, map,
                                olat, T, H, out, dev_status);
    }
    using P = proj::UpPlan<proj::kOlatBlock, 4>;
    cudaError_t e = cudaFuncSetAttribute(proj::upproj_kernel<proj::kOlatBlock, 4>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, P::kSmemBytes);
    if (e != cudaSuccess) return e;
    const dim3 grid(H, (T + proj::kOlatBlock - 1) / proj::kOlatBlock);
    return proj::launch_pdl(proj::upproj_kernel<proj::kOlatBlock, 4>, grid, proj::kUpThreads, P::kSmemBytes, stream,
                            map, olat, T, H, out, dev_status);
}

}  // namespace mla
