// Absorbed MLA decode for groups of at most 32 query rows (few heads), one SM per work unit.
//
// What is computed is the attend phase of mla_decode ("两张账" page, "第一张账"; MLA explainer section
// 2.2.2): every query row scores all its visible cached rows [c_t | k^R_t] with [q_abs | q^R] (576-wide),
// takes an online softmax and aggregates the latent c_t (512-wide), per piece of a sequence.
//
// With n_q * H <= 32 rows the CTA-pair kernel's 128-row MMAs would carry at most a quarter live rows,
// while its output accumulator still fills an SM's tensor memory.  Here both contractions are taken
// transposed, with the 128 tokens of a cache block as the M side:
//   S^T[token, row]   = K_block . Q^T   M = 128 tokens (A: the block's nine chunks as they stand, K-major),
//                                       N = NR rows (B: the query rows in shared memory), K = 576: 36 MMAs
//   O^T[latent, row] += V^T . P^T      M = 128 latent columns per block of four (A: the same chunks read
//                                       MN-major), N = NR rows (B: P rows in shared memory), K = 128 tokens:
//                                       32 MMAs
// so the two score buffers (NR columns each) and O^T (4 x NR columns) take 6 NR columns of tensor memory
// and one SM does the whole tile: each cache block is read from HBM once, by one SM, and nothing crosses
// SMs.  NR = 16 or 32 (the rows rounded up).
//
// Softmax: a thread per token (tensor-memory lane).  Row maxima by a warp reduction and an exchange of
// the four warps' maxima through shared memory; the running maximum is stale (it moves only when a tile's
// maximum exceeds it by more than 2^8, and then O^T is rescaled in tensor memory); each thread keeps its
// token lane's share of every row sum, and the shares are added once per segment.  P goes to shared
// memory as bf16 in the swizzled K-major layout of the second MMA's B operand.
//
// Scheduling and output are those of the pair kernel: the (sequence, tile) space is cut into equal
// contiguous ranges, one per CTA; a range yields pieces of sequences (segments), and each segment writes
// its unnormalised O (in the [column group][row] order of the workspace) and its (max, sum) per row for
// the merge kernel.
//
// Warp roles: warps 0..3 softmax and segment epilogue, warp 4 lane 0 bulk copies (a tile-aligned ring of
// three 48 KB slots = one block), warp 5 the MMAs.  Every wait is bounded: on expiry the kernel records
// MLA_DEVERR_TIMEOUT, leaves its loops, lets in-flight copies and MMAs land and frees tensor memory.
#include <cuda.h>
#include <math_constants.h>

#include <mutex>

#include "mla_internal.cuh"
#include "sm100.cuh"

namespace mla {
using namespace sm100;

namespace sm1 {

constexpr int kTile = kBlockTokens;               // tokens per tile = one cache block (128)
constexpr int kChunk = kTile * 128;               // [128 tokens x 64 columns] bf16 = 16 KB
constexpr int kCopyBytes = 3 * kChunk;            // 48 KB: three chunks per bulk copy
constexpr int kSlots = 3;                         // ring slots = one block: chunk c of a tile at c * 16 KB
constexpr int kThreads = 192;
constexpr int kSoftThreads = 128;
constexpr int kWarpProducer = 4, kWarpMma = 5;
constexpr uint32_t kNbRed = 1;                    // named barrier of the four softmax warps
constexpr uint64_t kLimitNs = 2000000000ull;      // 2 s per wait
constexpr float kRescaleLog2 = 8.0f;

// barriers
constexpr int kBFull = 0, kBEmpty = kSlots, kBSFull = 2 * kSlots, kBSEmpty = kBSFull + 2, kBPReady = kBSEmpty + 2,
              kBPFree = kBPReady + 2, kBQReady = kBPFree + 2, kBSegDone = kBQReady + 1, kBOFree = kBSegDone + 1,
              kBFin = kBOFree + 1, kNumBars = kBFin + 1;

template <int NR>
struct Lay {
    static constexpr int kOffRing = 0;
    static constexpr int kQChunk = NR * 128;                 // [NR rows x 64 columns] swizzled
    static constexpr int kOffQ = kSlots * kCopyBytes;        // nine query chunks
    static constexpr int kPChunk = NR * 128;                 // [NR rows x 64 tokens] swizzled
    static constexpr int kOffP = kOffQ + 9 * kQChunk;        // two P buffers of two chunks
    static constexpr int kOffRed = kOffP + 4 * kPChunk;      // [2][4 warps][NR] row maxima, [4][NR] row sums
    static constexpr int kOffBar = kOffRed + 3 * 4 * NR * 4;
    static constexpr int kOffTail = kOffBar + kNumBars * 8;  // tmem base, abort flag, tile total, first seq
    static constexpr int kSmemBytes = kOffTail + 32;
    static_assert(kOffQ % 1024 == 0 && kQChunk % 1024 == 0 && kOffP % 1024 == 0 && kPChunk % 1024 == 0,
                  "swizzle atoms 1024-aligned");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static constexpr uint32_t kTmemCols = 6 * NR <= 128 ? 128 : 256;
    __host__ __device__ static constexpr uint32_t col_s(uint32_t sb) { return sb * NR; }
    __host__ __device__ static constexpr uint32_t col_o(uint32_t mb) { return 2 * NR + mb * NR; }
};

struct Params {
    const uint16_t* q;
    const uint8_t* cache;
    const int32_t* block_table;
    const int32_t* kv_len;
    float* o_part;    // [slots][128 column groups of 4][rs rows] x float4
    float2* ml_part;  // [slots][rs]
    int32_t* dev_status;
    int64_t cap_blocks;
    int max_blocks;
    int B, n_q, H, R, P_g, slots, rs;
    float scale_log2;
};

__device__ __forceinline__ int seq_tiles(const Params& p, int b) {
    return valid_seq_tiles(p.kv_len[b], p.n_q, p.max_blocks);
}

struct Seg {
    int b, t0, t1, L, slot;
    const int32_t* tab;
};

__device__ __forceinline__ const uint8_t* tile_src(const Params& p, int32_t e) {
    if (e < 0 || e >= p.cap_blocks) {
        if (p.dev_status) atomicOr(p.dev_status, MLA_DEVERR_ROW_RANGE);
        e = 0;
    }
    return p.cache + static_cast<int64_t>(e) * kBlockBytes;
}

struct SegWalk {
    int b, tb, lo, hi, pidx;
    __device__ void init(int b0, int tb0, int lo_, int hi_, int pidx_) {
        lo = lo_;
        hi = hi_;
        pidx = pidx_;
        b = b0;
        tb = tb0;
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
                s.tab = p.block_table + static_cast<int64_t>(cb) * p.max_blocks;
                s.slot = cb + pidx;
                return true;
            }
        }
        return false;
    }
};

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int32_t* dev_status) {
    *abort_flag = 1;
    if (dev_status) atomicOr(dev_status, MLA_DEVERR_TIMEOUT);
}

// Maximum over the warp's 32 lanes (sm_100a warp reduction; inputs are finite or -inf).
__device__ __forceinline__ float warp_max_f32(float v) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}

template <int NR>
__device__ __forceinline__ void tmem_ld_rows(uint32_t taddr, float (&v)[NR]) {
    uint32_t r[32];
    if constexpr (NR == 16) tmem_ld16(taddr, r);
    else tmem_ld32(taddr, r);
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < NR; ++k) v[k] = __uint_as_float(r[k]);
}

template <int NR>
__global__ void __launch_bounds__(kThreads, 1) decode_sm_kernel(const Params p) {
    using L = Lay<NR>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffTail);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffTail + 4);
    int* nt_total = reinterpret_cast<int*>(smem + L::kOffTail + 8);
    int* walk0 = reinterpret_cast<int*>(smem + L::kOffTail + 12);
    volatile int never = 0;

    if ((sbase & 1023u) != 0) {
        if (tid == 0 && p.dev_status) atomicOr(p.dev_status, MLA_DEVERR_TIMEOUT);
        return;
    }
    if (tid == 0) {
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(&bars[kBFull + i], 1);
            mbar_init(&bars[kBEmpty + i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[kBSFull + i], 1);
            mbar_init(&bars[kBSEmpty + i], kSoftThreads);
            mbar_init(&bars[kBPReady + i], kSoftThreads);
            mbar_init(&bars[kBPFree + i], 1);
        }
        mbar_init(&bars[kBQReady], kSoftThreads);
        mbar_init(&bars[kBSegDone], 1);
        mbar_init(&bars[kBOFree], kSoftThreads);
        mbar_init(&bars[kBFin], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpProducer) tmem_alloc(tmem_slot, L::kTmemCols);
    // everything above touches only this CTA's own resources; inputs are read after this wait
    grid_dependency_wait();
    if (warp == 0) {
        // total tiles, then (by a warp scan) the sequence holding this CTA's first tile
        int s = 0;
        for (int b = lane; b < p.B; b += 32) {
            s += seq_tiles(p, b);
            if (blockIdx.x == 0 && p.dev_status) {
                const int Lb = p.kv_len[b];
                if (Lb < p.n_q) atomicOr(p.dev_status, MLA_DEVERR_KV_LEN);
                else if ((Lb + kTile - 1) / kTile > p.max_blocks) atomicOr(p.dev_status, MLA_DEVERR_ROW_RANGE);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const int lo0 = static_cast<int>((static_cast<int64_t>(blockIdx.x) * s) / p.P_g);
        int b0 = p.B, tb0 = s, run = 0;
        for (int base = 0; base < p.B; base += 32) {
            const int b = base + lane;
            const int nt = b < p.B ? seq_tiles(p, b) : 0;
            int inc = nt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += v;
            }
            const unsigned hit = __ballot_sync(0xffffffffu, b < p.B && run + inc > lo0);
            if (hit) {
                const int f = __ffs(hit) - 1;
                b0 = base + f;
                tb0 = run + __shfl_sync(0xffffffffu, inc - nt, f);
                break;
            }
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) {
            *nt_total = s;
            walk0[0] = b0;
            walk0[1] = tb0;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int Nt = *nt_total;
    const int pidx = static_cast<int>(blockIdx.x);
    const int lo = static_cast<int>((static_cast<int64_t>(pidx) * Nt) / p.P_g);
    const int hi = static_cast<int>((static_cast<int64_t>(pidx + 1) * Nt) / p.P_g);
    const int wb0 = walk0[0], wtb0 = walk0[1];

    if (warp == kWarpProducer) {
        // ---- copy producer: each block (144 KB, already in the operand layout) as three 48 KB bulk
        //      copies into the three ring slots; the block is read by this SM only, once
        if (lane == 0) {
            SegWalk w;
            w.init(wb0, wtb0, lo, hi, pidx);
            Seg s;
            uint32_t n = 0;  // tiles issued
            bool ok = true;
            const uint64_t once = l2_policy_evict_first();
            while (ok && w.next(p, s)) {
                for (int t = s.t0; ok && t < s.t1; ++t, ++n) {
                    const uint8_t* src = tile_src(p, s.tab[t]);
                    for (int k = 0; k < kSlots; ++k) {
                        ok = mbar_wait(&bars[kBEmpty + k], (n & 1u) ^ 1u, abort_flag, kLimitNs);
                        if (!ok) break;
                        mbar_arrive_expect_tx(&bars[kBFull + k], kCopyBytes);
                        bulk_load_hint(sbase + L::kOffRing + k * kCopyBytes, src + k * kCopyBytes, kCopyBytes,
                                       &bars[kBFull + k], once);
                    }
                }
            }
            if (!ok) raise_abort(abort_flag, p.dev_status);
            // let every issued copy land before the CTA can exit
            if (n > 0)
                for (int k = 0; k < kSlots; ++k) mbar_wait(&bars[kBFull + k], (n - 1) & 1u, &never, kLimitNs);
        }
    } else if (warp == kWarpMma) {
        // ---- MMA issuer: lane 0 issues, the warp zeroes V rows past a sequence's end
        constexpr uint32_t idesc_s = idesc_bf16_f32(128, NR, false, false);
        constexpr uint32_t idesc_o = idesc_bf16_f32(128, NR, true, false);
        const uint64_t ring_desc = sdesc_sw128(sbase + L::kOffRing, 16, 1024);          // K-major chunks
        const uint64_t v_desc = sdesc_sw128(sbase + L::kOffRing, kChunk, 1024);         // MN-major, 16 KB atoms
        const uint64_t q_desc = sdesc_sw128(sbase + L::kOffQ, 16, 1024);
        const uint64_t p_desc = sdesc_sw128(sbase + L::kOffP, 16, 1024);
        SegWalk w;
        w.init(wb0, wtb0, lo, hi, pidx);
        Seg s;
        uint32_t n = 0, kseg = 0;
        bool ok = true;
        while (ok && w.next(p, s)) {
            if (lane == 0) ok = mbar_wait(&bars[kBQReady], kseg & 1u, abort_flag, kLimitNs);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            for (int t = s.t0; ok && t < s.t1; ++t, ++n) {
                const uint32_t sb = n & 1u, us = n >> 1;
                const bool first = (t == s.t0);
                const int nvalid = min(kTile, s.L - t * kTile);
                if (lane == 0) {
                    ok = mbar_wait(&bars[kBSEmpty + sb], (us & 1u) ^ 1u, abort_flag, kLimitNs);
                    // a partial block waits for all three copies (its V rows past the end are zeroed first);
                    // a full one starts each copy's 12 MMAs as soon as that copy has landed
                    for (int k = 0; ok && nvalid < kTile && k < kSlots; ++k)
                        ok = mbar_wait(&bars[kBFull + k], n & 1u, abort_flag, kLimitNs);
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (nvalid < kTile) {
                    // rows past the sequence end: P is 0 there, make V 0 too (no 0 * NaN); their scores are masked
                    const int nz = (kTile - nvalid) * 8;  // 16-byte units per chunk
                    for (int i = lane; i < 8 * nz; i += 32) {
                        const int c = i / nz, u = i % nz;
                        *reinterpret_cast<uint4*>(smem + L::kOffRing + c * kChunk + nvalid * 128 + u * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_cta();
                }
                __syncwarp();
                if (lane == 0) {
                    // S^T = K Q^T into score buffer sb
                    const uint32_t d = tmem + L::col_s(sb);
                    for (int k = 0; ok && k < kSlots; ++k) {
                        if (nvalid == kTile) ok = mbar_wait(&bars[kBFull + k], n & 1u, abort_flag, kLimitNs);
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll
                        for (int j = 0; j < 3; ++j)
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                const int c = 3 * k + j;
                                mma_ss(d, ring_desc + static_cast<uint64_t>((c * kChunk + kk * 32) >> 4),
                                       q_desc + static_cast<uint64_t>((c * L::kQChunk + kk * 32) >> 4), idesc_s,
                                       (c | kk) ? 1u : 0u);
                            }
                    }
                    if (ok) mma_commit(smem_u32(&bars[kBSFull + sb]));
                    // O^T += V^T P^T once the softmax has staged P (and, at a segment's first tile, the
                    // epilogue has read the previous segment's O^T)
                    ok = ok && mbar_wait(&bars[kBPReady + sb], us & 1u, abort_flag, kLimitNs);
                    if (ok && first) ok = mbar_wait(&bars[kBOFree], (kseg & 1u) ^ 1u, abort_flag, kLimitNs);
                    if (ok) {
                        tc_fence_after();
                        const uint64_t pd = p_desc + static_cast<uint64_t>((sb * 2 * L::kPChunk) >> 4);
#pragma unroll
                        for (int mb = 0; mb < 4; ++mb) {
                            const uint64_t vd = v_desc + static_cast<uint64_t>((2 * mb * kChunk) >> 4);
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                mma_ss(tmem + L::col_o(mb), vd + static_cast<uint64_t>((kk * 2048) >> 4),
                                       pd + static_cast<uint64_t>(((kk >> 2) * L::kPChunk + (kk & 3) * 32) >> 4),
                                       idesc_o, (first && kk == 0) ? 0u : 1u);
                            // chunks 0..2 are slot 0, 3..5 slot 1, 6..8 slot 2
                            if (mb >= 1) mma_commit(smem_u32(&bars[kBEmpty + (mb - 1)]));
                        }
                        mma_commit(smem_u32(&bars[kBPFree + sb]));
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
            }
            if (lane == 0) mma_commit(smem_u32(&bars[kBSegDone]));  // the segment's O^T is complete
            __syncwarp();
            ++kseg;
        }
        if (!ok && lane == 0) raise_abort(abort_flag, p.dev_status);
        if (lane == 0) {
            mma_commit(smem_u32(&bars[kBFin]));
            mbar_wait(&bars[kBFin], 0, &never, kLimitNs);
        }
        __syncwarp();
    } else {
        // ---- softmax and segment epilogue: thread tk owns tensor-memory lane tk = token tk of a tile
        const int tk = tid;
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(32 * warp) << 16);
        float* red = reinterpret_cast<float*>(smem + L::kOffRed);  // [2][4][NR] maxima, then [4][NR] sums
        SegWalk w;
        w.init(wb0, wtb0, lo, hi, pidx);
        Seg s;
        uint32_t n = 0, kseg = 0;
        bool failed = false;
        while (!failed && w.next(p, s)) {
            // the segment's query rows: row r of sequence b is q[b * R + r]; 72 16-byte units per row into
            // nine swizzled chunks; rows R .. NR-1 are zero.  The previous segment's MMAs are all done
            // (its epilogue waited for them), so the query buffer is free.
            {
                constexpr int kUnits = NR * 72;
#pragma unroll
                for (int base = 0; base < kUnits; base += 9 * kSoftThreads) {
                    uint4 x[9];
#pragma unroll
                    for (int k = 0; k < 9; ++k) {
                        const int i = base + tid + k * kSoftThreads, r = i / 72, u = i % 72;
                        x[k] = make_uint4(0, 0, 0, 0);
                        if (i < kUnits && r < p.R)
                            x[k] = reinterpret_cast<const uint4*>(p.q + (static_cast<int64_t>(s.b) * p.R + r) * kRow)[u];
                    }
#pragma unroll
                    for (int k = 0; k < 9; ++k) {
                        const int i = base + tid + k * kSoftThreads, r = i / 72, u = i % 72;
                        if (i < kUnits)
                            *reinterpret_cast<uint4*>(smem + L::kOffQ + (u >> 3) * L::kQChunk + r * 128 +
                                                      (((u & 7) ^ (r & 7)) << 4)) = x[k];
                    }
                }
            }
            fence_proxy_async_cta();
            tc_fence_before();
            mbar_arrive(&bars[kBQReady]);
            // visible keys of row r (query j = r / H): 0 .. L - n_q + j
            float m[NR], lp[NR];
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                m[r] = -CUDART_INF_F;
                lp[r] = 0.f;
            }
            const int lim0 = s.L - p.n_q + 1;  // keys below this are visible to every query of the step
            for (int t = s.t0; t < s.t1; ++t, ++n) {
                const uint32_t sb = n & 1u, us = n >> 1;
                bool ok = mbar_wait(&bars[kBSFull + sb], us & 1u, abort_flag, kLimitNs);
                __syncwarp();
                tc_fence_after();
                float sv[NR];
                tmem_ld_rows<NR>(t_lane + L::col_s(sb), sv);
                tc_fence_before();
                mbar_arrive(&bars[kBSEmpty + sb]);
                const int tok = t * kTile + tk;
                if (tok < lim0) {
#pragma unroll
                    for (int r = 0; r < NR; ++r) sv[r] = r < p.R ? sv[r] : -CUDART_INF_F;
                } else {
#pragma unroll
                    for (int r = 0; r < NR; ++r) sv[r] = (r < p.R && tok < lim0 + r / p.H) ? sv[r] : -CUDART_INF_F;
                }
                // row maxima over the tile's 128 tokens: warp shuffles, then the four warps' maxima
                float* rmax = red + sb * 4 * NR;
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const float v = warp_max_f32(sv[r]);
                    if (lane == 0) rmax[warp * NR + r] = v;
                }
                if (bar_red_or(kNbRed, kSoftThreads, !ok || *abort_flag != 0)) {
                    failed = true;
                    break;
                }
                float alpha[NR];
                bool resc = false;
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const float tmax = fmaxf(fmaxf(rmax[r], rmax[NR + r]), fmaxf(rmax[2 * NR + r], rmax[3 * NR + r])) *
                                       p.scale_log2;
                    alpha[r] = 1.f;
                    if (tmax > m[r] + kRescaleLog2) {
                        alpha[r] = (m[r] == -CUDART_INF_F) ? 0.f : ex2_approx(m[r] - tmax);
                        m[r] = tmax;
                        resc = true;
                    }
                }
                uint32_t pk[NR / 2];
#pragma unroll
                for (int r = 0; r < NR; r += 2) {
                    const float p0 = ex2_approx(fmaf(sv[r], p.scale_log2, m[r] == -CUDART_INF_F ? 0.f : -m[r]));
                    const float p1 =
                        ex2_approx(fmaf(sv[r + 1], p.scale_log2, m[r + 1] == -CUDART_INF_F ? 0.f : -m[r + 1]));
                    lp[r] = fmaf(lp[r], alpha[r], p0);
                    lp[r + 1] = fmaf(lp[r + 1], alpha[r + 1], p1);
                    pk[r / 2] = cvt_bf16x2(p0, p1);
                }
                if (resc && t != s.t0) {
                    // the running max moved: rescale O^T's columns once the previous tile's MMAs are done (a
                    // segment's first tile starts O^T afresh)
                    ok = mbar_wait(&bars[kBPFree + (sb ^ 1u)], ((n - 1) >> 1) & 1u, abort_flag, kLimitNs);
                    __syncwarp();
                    tc_fence_after();
#pragma unroll 1
                    for (int mb = 0; mb < 4; ++mb) {
                        float v[NR];
                        tmem_ld_rows<NR>(t_lane + L::col_o(mb), v);
                        uint32_t o[32];
#pragma unroll
                        for (int r = 0; r < NR; ++r) o[r] = __float_as_uint(v[r] * alpha[r]);
                        if constexpr (NR == 16) tmem_st16(t_lane + L::col_o(mb), o);
                        else tmem_st32(t_lane + L::col_o(mb), o);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    if (!ok) raise_abort(abort_flag, p.dev_status);
                }
                // P of this tile into buffer sb, once the MMAs of tile n - 2 (same buffer) are done:
                // element (row r, token tk) of chunk tk / 64 at row r, unit ((tk % 64) / 8) ^ (r % 8)
                ok = mbar_wait(&bars[kBPFree + sb], (us & 1u) ^ 1u, abort_flag, kLimitNs);
                if (!ok) raise_abort(abort_flag, p.dev_status);
                uint8_t* pb = smem + L::kOffP + sb * 2 * L::kPChunk + (tk >> 6) * L::kPChunk + (tk & 7) * 2;
                const int tu = (tk & 63) >> 3;
#pragma unroll
                for (int r = 0; r < NR; r += 2) {
                    *reinterpret_cast<uint16_t*>(pb + r * 128 + ((tu ^ (r & 7)) << 4)) =
                        static_cast<uint16_t>(pk[r / 2] & 0xFFFFu);
                    *reinterpret_cast<uint16_t*>(pb + (r + 1) * 128 + ((tu ^ ((r + 1) & 7)) << 4)) =
                        static_cast<uint16_t>(pk[r / 2] >> 16);
                }
                fence_proxy_async_cta();
                mbar_arrive(&bars[kBPReady + sb]);
            }
            if (failed) break;
            // ---- segment epilogue: row sums over the 128 token lanes, then (max, sum) and O^T out
            float* rsum = red + 2 * 4 * NR;
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                float v = lp[r];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) rsum[warp * NR + r] = v;
            }
            const bool done = mbar_wait(&bars[kBSegDone], kseg & 1u, abort_flag, kLimitNs);
            if (bar_red_or(kNbRed, kSoftThreads, !done || *abort_flag != 0)) {
                failed = true;
                break;
            }
            tc_fence_after();
            if (tk < p.R) {
                float mm = 0.f;
#pragma unroll
                for (int r = 0; r < NR; ++r)
                    if (r == tk) mm = m[r];
                const float l = rsum[tk] + rsum[NR + tk] + rsum[2 * NR + tk] + rsum[3 * NR + tk];
                p.ml_part[static_cast<int64_t>(s.slot) * p.rs + tk] = make_float2(mm, l);
            }
            // O^T: lane = latent column c = 128 mb + 32 warp + lane, column r = row; the workspace holds
            // [column group c / 4][row] x float4, rs rows per slot
            float* oseg = p.o_part + static_cast<int64_t>(s.slot) * p.rs * kDc;
#pragma unroll 1
            for (int mb = 0; mb < 4; ++mb) {
                float v[NR];
                tmem_ld_rows<NR>(t_lane + L::col_o(mb), v);
                const int c = 128 * mb + 32 * warp + lane;
#pragma unroll
                for (int r = 0; r < NR; ++r)
                    if (r < p.R) oseg[((c >> 2) * p.rs + r) * 4 + (c & 3)] = v[r];
            }
            tc_fence_before();
            mbar_arrive(&bars[kBOFree]);
            // the sums area is rewritten by the next segment's epilogue only after its tiles' barriers
            ++kseg;
        }
        if (failed && tid == 0) raise_abort(abort_flag, p.dev_status);
    }

    // ------------------------------------------------------------------ teardown
    grid_dependents_launch();  // the merge kernel may be scheduled; it waits for this grid to finish
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpProducer) {
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    }
}

template <int NR>
cudaError_t launch(const Params& prm, cudaStream_t stream) {
    using L = Lay<NR>;
    cudaError_t e = cudaFuncSetAttribute(decode_sm_kernel<NR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(prm.P_g);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_sm_kernel<NR>, prm);
}

}  // namespace sm1

// Co-resident CTAs of the kernel on the current device (one per SM), at most kMaxSmCtas (the workspace
// has a slot per CTA).  The occupancy query runs once per device; the table is guarded for concurrent
// callers.
int decode_sm_ctas() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] > 0) return cache[dev];
    using L = sm1::Lay<32>;  // the larger layout bounds both
    if (cudaFuncSetAttribute(sm1::decode_sm_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             L::kSmemBytes) != cudaSuccess)
        return 0;
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sm1::decode_sm_kernel<32>, sm1::kThreads,
                                                      L::kSmemBytes) != cudaSuccess ||
        per_sm <= 0)
        return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return 0;
    const int n = per_sm * sms;
    cache[dev] = n < kMaxSmCtas ? n : kMaxSmCtas;
    return cache[dev];
}

cudaError_t launch_decode_sm(const uint16_t* q, const uint8_t* cache, int64_t cap_blocks, const int32_t* block_table,
                             int max_blocks, const int32_t* kv_len, int B, int n_q, int H, float scale, int ctas,
                             float* o_part, float2* ml_part, int slots, int rs, int32_t* dev_status,
                             cudaStream_t stream) {
    const int R = n_q * H;
    if (R < 1 || R > kMaxSmRows || R > rs || ctas < 1 || ctas > kMaxSmCtas || B + ctas > slots)
        return cudaErrorInvalidValue;
    sm1::Params prm;
    prm.q = q;
    prm.cache = cache;
    prm.block_table = block_table;
    prm.kv_len = kv_len;
    prm.o_part = o_part;
    prm.ml_part = ml_part;
    prm.dev_status = dev_status;
    prm.cap_blocks = cap_blocks;
    prm.max_blocks = max_blocks;
    prm.B = B;
    prm.n_q = n_q;
    prm.H = H;
    prm.R = R;
    prm.P_g = ctas;
    prm.slots = slots;
    prm.rs = rs;
    prm.scale_log2 = scale * 1.44269504088896340736f;
    return R <= 16 ? sm1::launch<16>(prm, stream) : sm1::launch<32>(prm, stream);
}

}  // namespace mla
