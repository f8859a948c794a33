// Absorbed MLA decode on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// What is computed ("两张账" page, "第一张账"; MLA explainer section 2.2.2):
// every query row (head h of query j of sequence b) scores all visible cached
// rows [c_t | k^R_t] with its absorbed query [q_abs | q^R] (576-wide inner
// product), takes a softmax and aggregates the latent c_t (512-wide):
// scores and aggregation both run against the one shared latent cache.
//
// Work split.  A cluster of two CTAs (one SM each) owns 128 query rows:
//   CTA 0 ("S"): the 128 absorbed query rows live in TMEM (the A operand, 288
//     columns); each 64-token tile of the cache is TMA-loaded (9 swizzled
//     [64 x 64] chunks) and S = Q K^T is formed by 36 tcgen05.mma (M=128,
//     N=64, K=16) into one of two TMEM score buffers.  Four warps (one thread
//     per query row) run the online softmax in fp32 and write P (bf16) straight
//     into CTA 1's shared memory over DSMEM.
//   CTA 1 ("O"): keeps the unnormalised latent output O[128 x 512] fp32 in its
//     whole TMEM and accumulates O += P V with 8 tcgen05.mma (M=128, N=256,
//     K=16) per tile; V is the first 512 columns of the same cache tile, read
//     as an MN-major operand.
// O for 128 rows x 512 fp32 fills an SM's 256 KB of TMEM, hence the pair.
//
// The softmax keeps a stale running max: it only rescales when a tile's max
// exceeds the running max by more than 2^8, so O in TMEM is rarely touched;
// rescales are done by CTA 1's epilogue warps on request.
//
// Scheduling: the kernel is persistent.  The (sequence, tile) space of all B
// sequences is cut into equal contiguous ranges, one per cluster (per row
// group of 128 rows), so every SM gets the same number of tiles whatever the
// length mix.  Each range yields one or more segments (pieces of sequences);
// a segment writes its unnormalised O and its (max, sum) to the workspace and
// mla_decode_finish merges the pieces of each sequence.
//
// Every wait is time-bounded: on expiry the kernel records MLA_DEVERR_TIMEOUT,
// both CTAs of the pair abandon their loops, let in-flight copies and MMAs
// land, free TMEM and return.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "mla_internal.cuh"
#include "sm100.cuh"

namespace mla {
using namespace sm100;

namespace tc {

constexpr int kTile = 64;           // tokens per tile
constexpr int kRows = 128;          // query rows per CTA pair
constexpr int kChunk = 64 * 64 * 2;  // [64 tokens x 64 columns] bf16 = 8 KB
constexpr int kKvChunks = 9;        // 576 / 64
constexpr int kVChunks = 8;         // 512 / 64
constexpr int kStagesS = 3;
constexpr int kStagesO = 3;
constexpr int kPBytes = kRows * kTile * 2;  // 16 KB bf16 P tile
constexpr int kThreads = 192;
constexpr uint64_t kLimitNs = 2000000000ull;  // 2 s per wait
constexpr float kRescaleLog2 = 8.0f;

// TMEM columns (512 allocated in each CTA)
constexpr uint32_t kColQ = 0;  // S CTA: Q rows, 288 columns of packed bf16 pairs
constexpr uint32_t kColS0 = 384;  // two 64-column score buffers: 384 and 448
__device__ __forceinline__ uint32_t col_s(uint32_t sb) { return kColS0 + 64u * sb; }

// shared memory layout (identical offsets in both CTAs so that mapa works)
constexpr int kOffKv = 0;                                    // S: 3 x 9 x 8 KB
constexpr int kOffV = 0;                                     // O: 3 x 8 x 8 KB
constexpr int kOffP = kStagesO * kVChunks * kChunk;          // O: 2 x 16 KB
constexpr int kOffAlpha = kOffP + 2 * kPBytes;               // O: 2 x 128 fp32
constexpr int kOffFlag = kOffAlpha + 2 * kRows * 4;          // O: 2 x u32
constexpr int kOffBar = kOffFlag + 16;                       // 16 mbarriers
constexpr int kOffTail = kOffBar + 16 * 8;                   // tmem base, abort, misc
constexpr int kSmemBytes = kOffTail + 32;
static_assert(kStagesS * kKvChunks * kChunk <= kOffBar, "S data overlaps barriers");
static_assert(kSmemBytes <= 232448, "shared memory budget");

// barrier slots
enum : int {
    // S CTA
    kBarKvFull = 0, kBarKvEmpty = 3, kBarSFull = 6, kBarSEmpty = 8, kBarPEmpty = 10, kBarQReady = 12,
    // O CTA
    kBarVFull = 0, kBarVEmpty = 3, kBarPFull = 6, kBarOFull = 8, kBarOFree = 9, kBarRescReq = 10,
    kBarRescDone = 11, kBarODrain = 12,
    // both
    kBarFin = 13
};

struct Params {
    const uint16_t* q;
    const int64_t* seq_start;
    const int32_t* kv_len;
    float* o_part;    // [G][slots][128][512]
    float2* ml_part;  // [G][slots][128]  (running max in log2 units, sum)
    int32_t* dev_status;
    int64_t cap;
    int B, n_q, H, R, G, P_g, slots;
    float scale_log2;
};

__device__ __forceinline__ int seq_tiles(const Params& p, int b) {
    const int L = p.kv_len[b];
    if (L < p.n_q) return 0;
    const int64_t s = p.seq_start[b];
    if (s < 0 || s + L > p.cap) return 0;
    return (L + kTile - 1) / kTile;
}

struct Seg {
    int b, t0, t1, L, slot;
    int64_t row0;
};

// Walks the segments of one cluster's tile range [lo, hi).
struct SegWalk {
    int b, tb, lo, hi, pidx;
    __device__ void init(const Params& p, int lo_, int hi_, int pidx_) {
        lo = lo_;
        hi = hi_;
        pidx = pidx_;
        b = 0;
        tb = 0;
        while (b < p.B) {
            const int nt = seq_tiles(p, b);
            if (tb + nt > lo) break;
            tb += nt;
            ++b;
        }
    }
    __device__ bool next(const Params& p, Seg& s) {
        while (b < p.B && tb < hi) {
            const int nt = seq_tiles(p, b);
            const int cb = b, ctb = tb;
            tb += nt;
            ++b;
            const int a = max(lo, ctb), e = min(hi, ctb + nt);
            if (a < e) {
                s.b = cb;
                s.t0 = a - ctb;
                s.t1 = e - ctb;
                s.L = p.kv_len[cb];
                s.row0 = p.seq_start[cb];
                s.slot = cb + pidx;
                return true;
            }
        }
        return false;
    }
};

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, uint32_t peer_abort, int32_t* dev_status) {
    *abort_flag = 1;
    st_cluster_u32(peer_abort, 1u);
    if (dev_status) atomicOr(dev_status, MLA_DEVERR_TIMEOUT);
}

__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap kv_map, const Params p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();  // 0: S CTA, 1: O CTA
    const uint32_t peer = rank ^ 1u;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTail);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffTail + 4);
    volatile int* resc_pb = reinterpret_cast<volatile int*>(smem + kOffTail + 8);
    int* nt_total = reinterpret_cast<int*>(smem + kOffTail + 12);
    volatile int never = 0;  // abort flag for teardown waits (never raised)

    if ((sbase & 1023u) != 0) {  // identical in both CTAs: both leave here
        if (tid == 0 && p.dev_status) atomicOr(p.dev_status, MLA_DEVERR_TIMEOUT);
        return;
    }
    if (tid == 0) {
        if (rank == 0) {
            for (int i = 0; i < kStagesS; ++i) {
                mbar_init(&bars[kBarKvFull + i], 1);
                mbar_init(&bars[kBarKvEmpty + i], 1);
            }
            for (int i = 0; i < 2; ++i) {
                mbar_init(&bars[kBarSFull + i], 1);
                mbar_init(&bars[kBarSEmpty + i], kRows);
                mbar_init(&bars[kBarPEmpty + i], 1);
            }
            mbar_init(&bars[kBarQReady], kRows);
        } else {
            for (int i = 0; i < kStagesO; ++i) {
                mbar_init(&bars[kBarVFull + i], 1);
                mbar_init(&bars[kBarVEmpty + i], 1);
            }
            for (int i = 0; i < 2; ++i) mbar_init(&bars[kBarPFull + i], kRows);
            mbar_init(&bars[kBarOFull], 1);
            mbar_init(&bars[kBarOFree], kRows);
            mbar_init(&bars[kBarRescReq], 1);
            mbar_init(&bars[kBarRescDone], kRows);
            mbar_init(&bars[kBarODrain], 1);
        }
        mbar_init(&bars[kBarFin], 1);
        *abort_flag = 0;
        *resc_pb = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        int s = 0;
        for (int b = lane; b < p.B; b += 32) {
            const int nt = seq_tiles(p, b);
            s += nt;
            if (blockIdx.x == 0 && p.dev_status) {
                const int L = p.kv_len[b];
                if (L < p.n_q) atomicOr(p.dev_status, MLA_DEVERR_KV_LEN);
                else if (p.seq_start[b] < 0 || p.seq_start[b] + L > p.cap) atomicOr(p.dev_status, MLA_DEVERR_ROW_RANGE);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) *nt_total = s;
    }
    if (warp == 4) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();  // peer barriers initialised before any remote arrive
    const uint32_t tmem = *tmem_slot;
    const int Nt = *nt_total;
    const int cid = static_cast<int>(blockIdx.x >> 1);
    const int g = cid / p.P_g, pidx = cid % p.P_g;
    const bool active = g < p.G;
    const int lo = static_cast<int>((static_cast<int64_t>(pidx) * Nt) / p.P_g);
    const int hi = static_cast<int>((static_cast<int64_t>(pidx + 1) * Nt) / p.P_g);
    const uint32_t peer_abort = mapa(sbase + kOffTail + 4, peer);
    const int64_t out_row_base = (static_cast<int64_t>(g) * p.slots) * kRows;

    if (active && rank == 0) {
        // =============================================================== S CTA
        if (warp == 4) {
            // ---- TMA producer: one 64-token tile = 9 chunks of [64 tokens x 64 cols]
            if (lane == 0) {
                prefetch_tmap(&kv_map);
                SegWalk w;
                w.init(p, lo, hi, pidx);
                Seg s;
                uint32_t n = 0;
                bool ok = true;
                while (ok && w.next(p, s)) {
                    for (int t = s.t0; t < s.t1; ++t, ++n) {
                        const uint32_t st = n % kStagesS, u = n / kStagesS;
                        if (!mbar_wait(&bars[kBarKvEmpty + st], (u & 1u) ^ 1u, abort_flag, kLimitNs)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&bars[kBarKvFull + st], kKvChunks * kChunk);
                        const int y = static_cast<int>(s.row0 + static_cast<int64_t>(t) * kTile);
#pragma unroll
                        for (int c = 0; c < kKvChunks; ++c)
                            tma_load_2d(sbase + kOffKv + (st * kKvChunks + c) * kChunk, &kv_map, 64 * c, y,
                                        &bars[kBarKvFull + st]);
                    }
                }
                if (!ok) raise_abort(abort_flag, peer_abort, p.dev_status);
                // let every issued copy land before the CTA can exit
                for (uint32_t i = (n > kStagesS ? n - kStagesS : 0); i < n; ++i)
                    mbar_wait(&bars[kBarKvFull + i % kStagesS], (i / kStagesS) & 1u, &never, kLimitNs);
            }
        } else if (warp == 5) {
            // ---- MMA issuer: S[sb] = Q K^T (A from TMEM, B = cache tile, K-major SW128)
            constexpr uint32_t idesc = idesc_bf16_f32(kRows, kTile, false, false);
            SegWalk w;
            w.init(p, lo, hi, pidx);
            Seg s;
            uint32_t n = 0, kseg = 0;
            bool ok = true;
            while (ok && w.next(p, s)) {
                ok = mbar_wait(&bars[kBarQReady], kseg & 1u, abort_flag, kLimitNs);
                ++kseg;
                for (int t = s.t0; ok && t < s.t1; ++t, ++n) {
                    const uint32_t st = n % kStagesS, u = n / kStagesS;
                    const uint32_t sb = n & 1u, us = n >> 1;
                    ok = mbar_wait(&bars[kBarKvFull + st], u & 1u, abort_flag, kLimitNs) &&
                         mbar_wait(&bars[kBarSEmpty + sb], (us & 1u) ^ 1u, abort_flag, kLimitNs);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t d = tmem + col_s(sb);
                        const uint32_t kv = sbase + kOffKv + st * kKvChunks * kChunk;
#pragma unroll
                        for (int k = 0; k < kRow / 16; ++k) {
                            const uint64_t bd = sdesc_sw128(kv + (k >> 2) * kChunk + (k & 3) * 32, 16, 1024);
                            mma_ts(d, tmem + kColQ + 8 * k, bd, idesc, k > 0 ? 1u : 0u);
                        }
                        mma_commit(smem_u32(&bars[kBarSFull + sb]));
                        mma_commit(smem_u32(&bars[kBarKvEmpty + st]));
                    }
                    __syncwarp();
                }
            }
            if (!ok && lane == 0) raise_abort(abort_flag, peer_abort, p.dev_status);
            if (lane == 0) mma_commit(smem_u32(&bars[kBarFin]));
            mbar_wait(&bars[kBarFin], 0, &never, kLimitNs);
        } else {
            // ---- softmax: warps 0..3, one thread per query row
            const int r = tid;
            const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
            const uint32_t peer_p = mapa(sbase + kOffP, peer);
            const uint32_t peer_alpha = mapa(sbase + kOffAlpha, peer);
            const uint32_t peer_flag = mapa(sbase + kOffFlag, peer);
            const uint32_t peer_pfull = mapa(smem_u32(&bars[kBarPFull]), peer);
            const int rr = g * kRows + r;
            const bool row_ok = rr < p.R;
            const int j = row_ok ? rr / p.H : 0;
            SegWalk w;
            w.init(p, lo, hi, pidx);
            Seg s;
            uint32_t n = 0;
            bool failed = false;
            while (!failed && w.next(p, s)) {
                // this segment's absorbed query row -> TMEM columns 0..287
                __syncwarp();
                const uint16_t* qrow = p.q + (static_cast<int64_t>(s.b) * p.R + (row_ok ? rr : 0)) * kRow;
#pragma unroll 1
                for (int c = 0; c < kKvChunks; ++c) {
                    uint32_t v[32];
                    const uint4* src = reinterpret_cast<const uint4*>(qrow + 64 * c);
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint4 x = row_ok ? src[k] : make_uint4(0, 0, 0, 0);
                        v[4 * k] = x.x;
                        v[4 * k + 1] = x.y;
                        v[4 * k + 2] = x.z;
                        v[4 * k + 3] = x.w;
                    }
                    tmem_st32(t_lane + kColQ + 32 * c, v);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars[kBarQReady]);
                const int lim = row_ok ? (s.L - p.n_q + j + 1) : 0;  // keys 0 .. lim-1 are visible
                float m = -CUDART_INF_F, l = 0.f;
                for (int t = s.t0; t < s.t1; ++t, ++n) {
                    const uint32_t sb = n & 1u, us = n >> 1;
                    bool ok = mbar_wait(&bars[kBarSFull + sb], us & 1u, abort_flag, kLimitNs);
                    __syncwarp();
                    tc_fence_after();
                    uint32_t a0[32], a1[32];
                    tmem_ld32(t_lane + col_s(sb), a0);
                    tmem_ld32(t_lane + col_s(sb) + 32, a1);
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(&bars[kBarSEmpty + sb]);
                    const int nvalid = max(0, min(kTile, lim - t * kTile));
                    float x[kTile];
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        x[k] = k < nvalid ? __uint_as_float(a0[k]) * p.scale_log2 : -CUDART_INF_F;
                        x[k + 32] = (k + 32) < nvalid ? __uint_as_float(a1[k]) * p.scale_log2 : -CUDART_INF_F;
                    }
                    float tmax = x[0];
#pragma unroll
                    for (int k = 1; k < kTile; ++k) tmax = fmaxf(tmax, x[k]);
                    const bool resc = tmax > m + kRescaleLog2;
                    float alpha = 1.f;
                    if (resc) {
                        alpha = (m == -CUDART_INF_F) ? 0.f : exp2f(m - tmax);
                        l *= alpha;
                        m = tmax;
                    }
                    const float mref = (m == -CUDART_INF_F) ? 0.f : m;
                    uint32_t pk[32];
                    float lsum = 0.f;
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        const float p0 = exp2f(x[2 * k] - mref), p1 = exp2f(x[2 * k + 1] - mref);
                        lsum += p0 + p1;
                        pk[k] = pack_bf16x2(p0, p1);
                    }
                    l += lsum;
                    ok = ok && mbar_wait<true>(&bars[kBarPEmpty + sb], (us & 1u) ^ 1u, abort_flag, kLimitNs);
                    if (bar_red_or(1, kRows, !ok || *abort_flag != 0)) {
                        failed = true;
                        break;
                    }
                    const bool flag = bar_red_or(2, kRows, resc && t != s.t0);
                    // P row r -> peer's P buffer (K-major, 128-byte swizzle: unit u at u ^ (r & 7))
                    const uint32_t prow = peer_p + sb * kPBytes + r * 128;
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        st_cluster_v4(prow + ((u ^ (r & 7)) << 4), pk[4 * u], pk[4 * u + 1], pk[4 * u + 2],
                                      pk[4 * u + 3]);
                    st_cluster_f32(peer_alpha + sb * kRows * 4 + 4 * r, alpha);
                    if (r == 0) st_cluster_u32(peer_flag + 4 * sb, flag ? 1u : 0u);
                    fence_proxy_async_cluster();
                    mbar_arrive_remote(peer_pfull + 8 * sb);
                }
                if (failed) break;
                if (row_ok) p.ml_part[out_row_base + static_cast<int64_t>(s.slot) * kRows + r] = make_float2(m, l);
            }
            if (failed && r == 0) raise_abort(abort_flag, peer_abort, p.dev_status);
        }
    } else if (active && rank == 1) {
        // =============================================================== O CTA
        if (warp == 4) {
            // ---- TMA producer: the 8 latent chunks of each tile (V)
            if (lane == 0) {
                prefetch_tmap(&kv_map);
                SegWalk w;
                w.init(p, lo, hi, pidx);
                Seg s;
                uint32_t n = 0;
                bool ok = true;
                while (ok && w.next(p, s)) {
                    for (int t = s.t0; t < s.t1; ++t, ++n) {
                        const uint32_t st = n % kStagesO, u = n / kStagesO;
                        if (!mbar_wait(&bars[kBarVEmpty + st], (u & 1u) ^ 1u, abort_flag, kLimitNs)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&bars[kBarVFull + st], kVChunks * kChunk);
                        const int y = static_cast<int>(s.row0 + static_cast<int64_t>(t) * kTile);
#pragma unroll
                        for (int c = 0; c < kVChunks; ++c)
                            tma_load_2d(sbase + kOffV + (st * kVChunks + c) * kChunk, &kv_map, 64 * c, y,
                                        &bars[kBarVFull + st]);
                    }
                }
                if (!ok) raise_abort(abort_flag, peer_abort, p.dev_status);
                for (uint32_t i = (n > kStagesO ? n - kStagesO : 0); i < n; ++i)
                    mbar_wait(&bars[kBarVFull + i % kStagesO], (i / kStagesO) & 1u, &never, kLimitNs);
            }
        } else if (warp == 5) {
            // ---- MMA issuer: O += P V (A = P, K-major SW128; B = V, MN-major SW128)
            constexpr uint32_t idesc = idesc_bf16_f32(kRows, 256, false, true);
            const uint32_t peer_pempty = mapa(smem_u32(&bars[kBarPEmpty]), peer);
            volatile uint32_t* flags = reinterpret_cast<volatile uint32_t*>(smem + kOffFlag);
            SegWalk w;
            w.init(p, lo, hi, pidx);
            Seg s;
            uint32_t n = 0, kseg = 0, nresc = 0;
            bool ok = true;
            while (ok && w.next(p, s)) {
                for (int t = s.t0; ok && t < s.t1; ++t, ++n) {
                    const uint32_t st = n % kStagesO, u = n / kStagesO;
                    const uint32_t pb = n & 1u, up = n >> 1;
                    const bool first = (t == s.t0);
                    ok = mbar_wait(&bars[kBarVFull + st], u & 1u, abort_flag, kLimitNs) &&
                         mbar_wait<true>(&bars[kBarPFull + pb], up & 1u, abort_flag, kLimitNs);
                    if (ok && first) ok = mbar_wait(&bars[kBarOFree], (kseg & 1u) ^ 1u, abort_flag, kLimitNs);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    if (!first && flags[pb] != 0u) {
                        // stale max moved: have the epilogue rescale O once all earlier MMAs are done
                        if (lane == 0) {
                            *resc_pb = static_cast<int>(pb);
                            mma_commit(smem_u32(&bars[kBarODrain]));
                            mbar_arrive(&bars[kBarRescReq]);
                        }
                        __syncwarp();
                        ok = __all_sync(0xffffffffu,
                                        mbar_wait(&bars[kBarRescDone], nresc & 1u, abort_flag, kLimitNs));
                        ++nresc;
                        if (!ok) break;
                    }
                    const int nvalid = min(kTile, s.L - t * kTile);
                    if (nvalid < kTile) {
                        // rows past the sequence end: P is 0 there, make V 0 too (no 0 * NaN)
                        uint8_t* vst = smem + kOffV + st * kVChunks * kChunk;
                        const int nz = (kTile - nvalid) * 8;  // 16-byte units per chunk
                        for (int i = lane; i < kVChunks * nz; i += 32) {
                            const int c = i / nz, k = i % nz;
                            *reinterpret_cast<uint4*>(vst + c * kChunk + nvalid * 128 + k * 16) = make_uint4(0, 0, 0, 0);
                        }
                        fence_proxy_async_cta();
                        __syncwarp();
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t pa = sbase + kOffP + pb * kPBytes;
                        const uint32_t vb = sbase + kOffV + st * kVChunks * kChunk;
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
#pragma unroll
                            for (int k = 0; k < kTile / 16; ++k) {
                                const uint64_t ad = sdesc_sw128(pa + k * 32, 16, 1024);
                                const uint64_t bd = sdesc_sw128(vb + (4 * half) * kChunk + k * 2048, kChunk, 1024);
                                mma_ss(tmem + 256 * half, ad, bd, idesc, (first && k == 0) ? 0u : 1u);
                            }
                        }
                        mma_commit(smem_u32(&bars[kBarVEmpty + st]));
                        mma_commit(peer_pempty + 8 * pb);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (lane == 0) mma_commit(smem_u32(&bars[kBarOFull]));
                __syncwarp();
                ++kseg;
            }
            if (!ok && lane == 0) raise_abort(abort_flag, peer_abort, p.dev_status);
            if (lane == 0) mma_commit(smem_u32(&bars[kBarFin]));
            mbar_wait(&bars[kBarFin], 0, &never, kLimitNs);
        } else {
            // ---- epilogue: warps 0..3, one thread per query row
            const int r = tid;
            const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
            const float* alphas = reinterpret_cast<const float*>(smem + kOffAlpha);
            const int rr = g * kRows + r;
            const bool row_ok = rr < p.R;
            SegWalk w;
            w.init(p, lo, hi, pidx);
            Seg s;
            uint32_t kseg = 0, nresc = 0;
            bool ok = true;
            while (ok && w.next(p, s)) {
                // serve rescale requests until this segment's O is complete.  Lane 0
                // polls; the warp then waits together so tcgen05.ld/st stay converged.
                const uint64_t t0 = globaltimer_ns();
                uint32_t it = 0;
                for (;;) {
                    int ev = 0;  // 1: O complete, 2: rescale request, 3: give up
                    if (lane == 0) {
                        if (mbar_test(smem_u32(&bars[kBarOFull]), kseg & 1u)) ev = 1;
                        else if (mbar_test(smem_u32(&bars[kBarRescReq]), nresc & 1u)) ev = 2;
                        else if (*abort_flag) ev = 3;
                        else if ((++it & 255u) == 0 && globaltimer_ns() - t0 > kLimitNs) ev = 3;
                    }
                    ev = __shfl_sync(0xffffffffu, ev, 0);
                    if (ev == 1) {
                        ok = mbar_wait(&bars[kBarOFull], kseg & 1u, abort_flag, kLimitNs);
                        break;
                    }
                    if (ev == 3) {
                        ok = false;
                        break;
                    }
                    if (ev == 2) {
                        ok = mbar_wait(&bars[kBarRescReq], nresc & 1u, abort_flag, kLimitNs) &&
                             mbar_wait(&bars[kBarODrain], nresc & 1u, abort_flag, kLimitNs);
                        __syncwarp();
                        tc_fence_after();
                        const float a = alphas[*resc_pb * kRows + r];
                        if (__any_sync(0xffffffffu, a != 1.f)) {
#pragma unroll 1
                            for (int c = 0; c < 16; ++c) {
                                uint32_t v[32];
                                tmem_ld32(t_lane + 32 * c, v);
                                tmem_wait_ld();
#pragma unroll
                                for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * a);
                                tmem_st32(t_lane + 32 * c, v);
                            }
                            tmem_wait_st();
                        }
                        tc_fence_before();
                        mbar_arrive(&bars[kBarRescDone]);
                        ++nresc;
                        if (!__all_sync(0xffffffffu, ok)) {
                            ok = false;
                            break;
                        }
                        continue;
                    }
                    __nanosleep(64);
                }
                ok = __all_sync(0xffffffffu, ok);
                __syncwarp();
                if (!ok) break;
                tc_fence_after();
                float* orow = p.o_part + (out_row_base + static_cast<int64_t>(s.slot) * kRows + r) * kDc;
#pragma unroll 1
                for (int c = 0; c < 16; ++c) {
                    uint32_t v[32];
                    tmem_ld32(t_lane + 32 * c, v);
                    tmem_wait_ld();
                    if (row_ok) {
                        float4* dst = reinterpret_cast<float4*>(orow + 32 * c);
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            dst[k] = make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                                 __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
                    }
                }
                tc_fence_before();
                mbar_arrive(&bars[kBarOFree]);
                ++kseg;
            }
            if (!ok && lane == 0) raise_abort(abort_flag, peer_abort, p.dev_status);
        }
    }

    // ------------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the peer no longer touches this CTA's shared memory
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
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

}  // namespace tc

int decode_tc_max_clusters() { return 74; }

// Co-resident clusters of the kernel on the current device (cached per device).
int decode_tc_clusters() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cache[dev] > 0) return cache[dev];
    if (cudaFuncSetAttribute(tc::decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::kSmemBytes) !=
        cudaSuccess)
        return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * decode_tc_max_clusters());
    cfg.blockDim = dim3(tc::kThreads);
    cfg.dynamicSmemBytes = tc::kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, tc::decode_tc_kernel, &cfg) != cudaSuccess || n <= 0) return 0;
    cache[dev] = n < decode_tc_max_clusters() ? n : decode_tc_max_clusters();
    return cache[dev];
}

cudaError_t launch_decode_tc(const uint16_t* q, const uint16_t* cache, int64_t cap, const int64_t* seq_start,
                             const int32_t* kv_len, int B, int n_q, int H, float scale, int clusters_per_group,
                             float* o_part, float2* ml_part, int slots, int32_t* dev_status, cudaStream_t stream) {
    const int R = n_q * H;
    const int G = (R + tc::kRows - 1) / tc::kRows;
    int total = decode_tc_clusters();
    if (total <= 0) return cudaErrorNotSupported;
    int P_g = total / G;
    if (P_g < 1) P_g = 1;
    if (clusters_per_group > 0 && clusters_per_group < P_g) P_g = clusters_per_group;
    if (B + P_g > slots) return cudaErrorInvalidValue;
    if (cudaFuncSetAttribute(tc::decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::kSmemBytes) !=
        cudaSuccess)
        return cudaErrorNotSupported;
    auto encode = tc::encode_fn();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap map;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(kRow), static_cast<cuuint64_t>(cap)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(kRow) * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(cache), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    tc::Params prm;
    prm.q = q;
    prm.seq_start = seq_start;
    prm.kv_len = kv_len;
    prm.o_part = o_part;
    prm.ml_part = ml_part;
    prm.dev_status = dev_status;
    prm.cap = cap;
    prm.B = B;
    prm.n_q = n_q;
    prm.H = H;
    prm.R = R;
    prm.G = G;
    prm.P_g = P_g;
    prm.slots = slots;
    prm.scale_log2 = scale * 1.44269504088896340736f;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * G * P_g);
    cfg.blockDim = dim3(tc::kThreads);
    cfg.dynamicSmemBytes = tc::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, tc::decode_tc_kernel, map, prm);
}

}  // namespace mla
