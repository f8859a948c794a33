// Absorbed MLA decode on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// What is computed ("两张账" page, "第一张账"; MLA explainer section 2.2.2):
// every query row (head h of query j of sequence b) scores all visible cached
// rows [c_t | k^R_t] with its absorbed query [q_abs | q^R] (576-wide inner
// product), takes a softmax and aggregates the latent c_t (512-wide):
// scores and aggregation both run against the one shared latent cache.
//
// Work split.  A cluster of two CTAs (one SM each) owns 128 query rows:
//   CTA 0 ("S"): the latent part of the 128 absorbed query rows lives in TMEM
//     (the A operand, 256 columns of packed bf16 pairs), the RoPE part in shared
//     memory.  Each 128-token cache block (9 pre-swizzled [128 x 64] chunks,
//     144 KB) arrives as three 48 KB bulk copies into a ring of three copy slots
//     (marked evict_last in L2, so that CTA 1's read of the same block hits L2),
//     and S = Q K^T is formed by 36 tcgen05.mma (M=128, N=128, K=16:
//     full-rate shape) into one of two TMEM score buffers.  Eight warps (a query
//     row's 128 scores split over two threads) run the online softmax in fp32
//     and stage P (bf16) in shared memory; a sender warp ships each staged P
//     tile to CTA 1 with a single bulk copy over DSMEM, so neither the copy nor
//     CTA 1's progress ever holds up the softmax.
//   CTA 1 ("O"): keeps the unnormalised latent output O[128 x 512] fp32 in its
//     whole TMEM and accumulates O += P V with 16 tcgen05.mma per tile (M=128,
//     N=256 per four latent chunks, K=16: the widest N re-reads P least often
//     from shared memory, whose bandwidth bounds this SM); V is the first 512
//     columns of the same cache block (its first 128 KB, two 64 KB bulk copies
//     into two stages), read as an MN-major operand.
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
#include <math_constants.h>

#include <mutex>

#include "mla_internal.cuh"
#include "sm100.cuh"

namespace mla {
using namespace sm100;

namespace tc {

constexpr int kTile = kBlockTokens;  // tokens per tile = one cache block (128)
constexpr int kRows = 128;           // query rows per CTA pair
constexpr int kChunk = kTile * 128;  // [128 tokens x 64 columns] bf16 = 16 KB
constexpr int kKvChunks = 9;         // 576 / 64
constexpr int kCopyChunks = 3;       // chunks per bulk copy (48 KB)
constexpr int kCopies = kKvChunks / kCopyChunks;  // S CTA: copies per tile
constexpr int kCopyBytes = kCopyChunks * kChunk;
constexpr int kRingSlots = 3;        // S CTA: ring of 48 KB copy slots (one tile)
constexpr int kVChunksPerStage = 4;  // O CTA: a V stage = 4 chunks (64 KB) = one N=256 MMA column block
constexpr int kVStageBytes = kVChunksPerStage * kChunk;
constexpr int kVPerTile = 8 / kVChunksPerStage;  // V stages per tile (the 8 latent chunks)
constexpr int kVStages = 2;          // O CTA: ring of V stages
constexpr int kPBytes = kRows * kTile * 2;       // 32 KB bf16 P tile: two [128 x 64] swizzled atoms
constexpr int kMsgBytes = kPBytes + kRows * 4;  // P | alpha[128] (per-row rescale factors): one bulk copy
constexpr int kMsgStride = 33792;    // 1024-aligned message slots (P atoms must start 1024-aligned)
constexpr int kPSlots = 3;           // O CTA: message slots, so P(t) can land while P V(t-2) still runs
constexpr int kSoftWarps = 8;        // S CTA: two warps per TMEM lane quadrant
constexpr int kSoftThreads = kSoftWarps * 32;
constexpr int kWarpProducer = 8, kWarpMma = 9, kWarpSender = 10;
constexpr int kThreads = 352;
constexpr int kSyncThreads = kSoftThreads + 32;  // softmax warps + the sender warp
// named barriers, S CTA: 1..4 the two warps of a TMEM lane quadrant; the rest over kSyncThreads
constexpr uint32_t kNbQFree = 5, kNbFail = 6, kNbStaged = 7, kNbStageFree = 8;
constexpr uint64_t kLimitNs = 2000000000ull;  // 2 s per wait
constexpr float kRescaleLog2 = 8.0f;
static_assert(kKvChunks % kCopyChunks == 0, "a tile is a whole number of copies");
static_assert(kTile == 128, "the MMA N and the P layout assume 128-token tiles");

// TMEM columns (512 allocated in each CTA)
constexpr uint32_t kColQ = 0;     // S CTA: latent Q rows, 256 columns of packed bf16 pairs
constexpr uint32_t kColS0 = 256;  // S CTA: two 128-column score buffers (256, 384)
__device__ __forceinline__ uint32_t col_s(uint32_t sb) { return kColS0 + 128u * sb; }

// shared memory, S CTA.  P messages are built in two staging buffers, so the softmax can stage P(t+1)
// while the copy of P(t) is still queued behind tile loads on this SM's copy engine; staging buffer 1
// shares its space with the Q transpose tiles, used only while a segment's queries are reloaded.
constexpr int kSOffRing = 0;                                  // 3 x 48 KB
constexpr int kSOffQR = kRingSlots * kCopyBytes;              // RoPE part of Q: [128 x 64] swizzled, 16 KB
constexpr int kSOffStage0 = kSOffQR + kRows * 128;            // P message staging buffer 0 (kMsgBytes)
constexpr int kSOffXchg = kSOffStage0 + kMsgStride;           // [2][128] fp32 half-row maxima / sums
constexpr int kSOffQT = kSOffXchg + 2 * kRows * 4;            // 8 warps x [32 rows x 128 B] Q transpose tiles
constexpr int kSOffStage1 = kSOffQT;                          //   = P message staging buffer 1
constexpr int kQTBytes = kSoftWarps * 32 * 128;
constexpr int kSOffBar = kSOffQT + (kQTBytes > kMsgBytes ? kQTBytes : kMsgBytes);
constexpr int kSBarFull = 0, kSBarEmpty = kRingSlots, kSBarSFull = 2 * kRingSlots, kSBarSEmpty = kSBarSFull + 2,
              kSBarPEmpty = kSBarSEmpty + 2, kSBarQReady = kSBarPEmpty + kPSlots, kSBarFin = kSBarQReady + 1,
              kSNumBars = kSBarFin + 1;
constexpr int kSOffTail = kSOffBar + kSNumBars * 8;
// shared memory, O CTA: the last message slot ends at its alpha values (no padding), barriers follow
constexpr int kOOffV = 0;                                     // 2 x 64 KB
constexpr int kOOffMsg = kVStages * kVStageBytes;             // kPSlots message slots, kMsgStride apart
constexpr int kOOffBar = kOOffMsg + (kPSlots - 1) * kMsgStride + kMsgBytes;
constexpr int kOBarVFull = 0, kOBarVEmpty = kVStages, kOBarPFull = 2 * kVStages, kOBarOFull = kOBarPFull + kPSlots,
              kOBarOFree = kOBarOFull + 1, kOBarRescReq = kOBarOFree + 1, kOBarRescDone = kOBarRescReq + 1,
              kOBarODrain = kOBarRescDone + 1, kOBarFin = kOBarODrain + 1, kONumBars = kOBarFin + 1;
constexpr int kOOffTail = kOOffBar + kONumBars * 8;
constexpr int kTailBytes = 32;  // tmem base, abort flag, resc slot, tile total, first sequence and its tile
constexpr int kSmemBytes = (kSOffTail > kOOffTail ? kSOffTail : kOOffTail) + kTailBytes;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kSOffQR % 1024 == 0 && kSOffStage0 % 1024 == 0 && kSOffStage1 % 1024 == 0 && kOOffMsg % 1024 == 0 &&
                  kMsgStride % 1024 == 0,
              "swizzle atoms 1024-aligned");
static_assert(kOOffBar % 8 == 0 && kSOffBar % 8 == 0, "mbarriers 8-byte aligned");
static_assert(kMsgBytes % 16 == 0, "bulk copy size");
static_assert(kMsgStride >= kMsgBytes, "message slot");

struct Params {
    const uint16_t* q;
    const uint8_t* cache;        // pool of blocks of kBlockBytes
    const int32_t* block_table;  // [B][max_blocks] pool block of each 128-token tile of a sequence
    const int32_t* kv_len;
    float* o_part;    // [G][slots][128 column groups of 4][128 rows] x float4 (unnormalised O)
    float2* ml_part;  // [G][slots][128]  (running max in log2 units, sum)
    int32_t* dev_status;
    int64_t cap_blocks;
    int max_blocks;
    int B, n_q, H, R, G, P_g, slots;
    float scale_log2;
};

__device__ __forceinline__ int seq_tiles(const Params& p, int b) {
    return valid_seq_tiles(p.kv_len[b], p.n_q, p.max_blocks);
}

struct Seg {
    int b, t0, t1, L, slot;
    const int32_t* tab;  // the sequence's row of the block table
};

// Pool block of tile t of a segment; an entry outside the pool is reported and replaced by block 0
// (that sequence's result is then unspecified, but no access leaves the pool).
__device__ __forceinline__ const uint8_t* tile_src(const Params& p, int32_t e) {
    if (e < 0 || e >= p.cap_blocks) {
        if (p.dev_status) atomicOr(p.dev_status, MLA_DEVERR_ROW_RANGE);
        e = 0;
    }
    return p.cache + static_cast<int64_t>(e) * kBlockBytes;
}

// Walks the segments of one cluster's tile range [lo, hi), starting at sequence b0 whose
// first tile has global index tb0 (found once per CTA in the prologue).
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

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, uint32_t peer_abort, int32_t* dev_status) {
    *abort_flag = 1;
    st_cluster_u32(peer_abort, 1u);
    if (dev_status) atomicOr(dev_status, MLA_DEVERR_TIMEOUT);
}

__device__ __forceinline__ float fmax64(const float (&v)[64]) {
    float a = fmaxf(v[0], v[1]), b = fmaxf(v[2], v[3]), c = fmaxf(v[4], v[5]), d = fmaxf(v[6], v[7]);
#pragma unroll
    for (int k = 8; k < 64; k += 4) {
        a = fmaxf(a, v[k]);
        b = fmaxf(b, v[k + 1]);
        c = fmaxf(c, v[k + 2]);
        d = fmaxf(d, v[k + 3]);
    }
    return fmaxf(fmaxf(a, b), fmaxf(c, d));
}

__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const Params p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();  // 0: S CTA, 1: O CTA
    const uint32_t peer = rank ^ 1u;
    const int tail = rank == 0 ? kSOffTail : kOOffTail;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (rank == 0 ? kSOffBar : kOOffBar));
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + tail);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + tail + 4);
    volatile int* resc_pb = reinterpret_cast<volatile int*>(smem + tail + 8);
    int* nt_total = reinterpret_cast<int*>(smem + tail + 12);
    int* walk0 = reinterpret_cast<int*>(smem + tail + 16);  // [first sequence of this cluster, its first tile]
    volatile int never = 0;  // abort flag for teardown waits (never raised)

    if ((sbase & 1023u) != 0) {  // identical in both CTAs: both leave here
        if (tid == 0 && p.dev_status) atomicOr(p.dev_status, MLA_DEVERR_TIMEOUT);
        return;
    }
    if (tid == 0) {
        if (rank == 0) {
            for (int i = 0; i < kRingSlots; ++i) {
                mbar_init(&bars[kSBarFull + i], 1);
                mbar_init(&bars[kSBarEmpty + i], 1);
            }
            for (int i = 0; i < 2; ++i) {
                mbar_init(&bars[kSBarSFull + i], 1);
                mbar_init(&bars[kSBarSEmpty + i], kSoftThreads);
            }
            for (int i = 0; i < kPSlots; ++i) mbar_init(&bars[kSBarPEmpty + i], 1);
            mbar_init(&bars[kSBarQReady], kSoftThreads);
            mbar_init(&bars[kSBarFin], 1);
        } else {
            for (int i = 0; i < kVStages; ++i) {
                mbar_init(&bars[kOBarVFull + i], 1);
                mbar_init(&bars[kOBarVEmpty + i], 1);
            }
            for (int i = 0; i < kPSlots; ++i) mbar_init(&bars[kOBarPFull + i], 1);
            mbar_init(&bars[kOBarOFull], 1);
            mbar_init(&bars[kOBarOFree], kRows);
            mbar_init(&bars[kOBarRescReq], 1);
            mbar_init(&bars[kOBarRescDone], kRows);
            mbar_init(&bars[kOBarODrain], 1);
            mbar_init(&bars[kOBarFin], 1);
        }
        *abort_flag = 0;
        *resc_pb = 0;
        fence_mbar_init();
    }
    if (warp == kWarpProducer) tmem_alloc(tmem_slot, 512);
    // Everything above touches only this CTA's own resources, so it overlaps the previous kernel's tail
    // under programmatic dependent launch; every read of the call's inputs comes after this wait.
    grid_dependency_wait();
    if (warp == 0) {
        // total tiles, then (by a warp scan) the sequence holding this cluster's first tile
        int s = 0;
        for (int b = lane; b < p.B; b += 32) {
            const int nt = seq_tiles(p, b);
            s += nt;
            if (blockIdx.x == 0 && p.dev_status) {
                const int L = p.kv_len[b];
                if (L < p.n_q) atomicOr(p.dev_status, MLA_DEVERR_KV_LEN);
                else if ((L + kTile - 1) / kTile > p.max_blocks) atomicOr(p.dev_status, MLA_DEVERR_ROW_RANGE);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const int pidx0 = static_cast<int>(blockIdx.x >> 1) % p.P_g;
        const int lo0 = static_cast<int>((static_cast<int64_t>(pidx0) * s) / p.P_g);
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
    cluster_sync();  // peer barriers initialised before any remote arrive
    const uint32_t tmem = *tmem_slot;
    const int Nt = *nt_total;
    const int cid = static_cast<int>(blockIdx.x >> 1);
    const int g = cid / p.P_g, pidx = cid % p.P_g;
    const bool active = g < p.G;
    const int lo = static_cast<int>((static_cast<int64_t>(pidx) * Nt) / p.P_g);
    const int hi = static_cast<int>((static_cast<int64_t>(pidx + 1) * Nt) / p.P_g);
    const int wb0 = walk0[0], wtb0 = walk0[1];
    const uint32_t peer_abort = mapa(sbase + (rank == 0 ? kOOffTail : kSOffTail) + 4, peer);
    const int64_t out_row_base = (static_cast<int64_t>(g) * p.slots) * kRows;

    if (active && rank == 0) {
        // =============================================================== S CTA
        if (warp == kWarpProducer) {
            // ---- copy producer: each 128-token block (144 KB, already in the operand layout)
            //      lands as three 48 KB bulk copies, one per ring slot, marked to stay in L2
            //      for the O CTA's read of the latent part.  (Pulling blocks into L2 ahead of
            //      the ring was measured to lose them to eviction and only add DRAM reads.)
            if (lane == 0) {
                SegWalk w;
                w.init(wb0, wtb0, lo, hi, pidx);
                Seg s;
                uint32_t nc = 0;  // copies issued
                bool ok = true;
                const uint64_t keep = l2_policy_evict_last();
                while (ok && w.next(p, s)) {
                    for (int t = s.t0; ok && t < s.t1; ++t) {
                        const uint8_t* src = tile_src(p, s.tab[t]);
                        for (int k = 0; k < kCopies; ++k, ++nc) {
                            const uint32_t slot = nc % kRingSlots, u = nc / kRingSlots;
                            ok = mbar_wait(&bars[kSBarEmpty + slot], (u & 1u) ^ 1u, abort_flag, kLimitNs);
                            if (!ok) break;
                            mbar_arrive_expect_tx(&bars[kSBarFull + slot], kCopyBytes);
                            bulk_load_hint(sbase + kSOffRing + slot * kCopyBytes, src + k * kCopyBytes, kCopyBytes,
                                           &bars[kSBarFull + slot], keep);
                        }
                    }
                }
                if (!ok) raise_abort(abort_flag, peer_abort, p.dev_status);
                // let every issued copy land before the CTA can exit
                for (uint32_t i = (nc > kRingSlots ? nc - kRingSlots : 0); i < nc; ++i)
                    mbar_wait(&bars[kSBarFull + i % kRingSlots], (i / kRingSlots) & 1u, &never, kLimitNs);
            }
        } else if (warp == kWarpMma) {
            // ---- MMA issuer (one thread): S[sb] = Q K^T.  Latent chunks: A from TMEM; the
            //      RoPE chunk: A = Q^R in shared memory.  B = cache chunks (K-major SW128,
            //      128 rows).  Each ring slot is released (commit) once its 12 MMAs finish.
            if (lane == 0) {
                constexpr uint32_t idesc = idesc_bf16_f32(kRows, kTile, false, false);
                const uint64_t ring_desc = sdesc_sw128(sbase + kSOffRing, 16, 1024);
                const uint64_t qr_desc = sdesc_sw128(sbase + kSOffQR, 16, 1024);
                SegWalk w;
                w.init(wb0, wtb0, lo, hi, pidx);
                Seg s;
                uint32_t n = 0, kseg = 0, nc = 0;
                bool ok = true;
                while (ok && w.next(p, s)) {
                    ok = mbar_wait(&bars[kSBarQReady], kseg & 1u, abort_flag, kLimitNs);
                    ++kseg;
                    for (int t = s.t0; ok && t < s.t1; ++t, ++n) {
                        const uint32_t sb = n & 1u, us = n >> 1;
                        ok = mbar_wait(&bars[kSBarSEmpty + sb], (us & 1u) ^ 1u, abort_flag, kLimitNs);
                        const uint32_t d = tmem + col_s(sb);
                        for (int k = 0; ok && k < kCopies; ++k, ++nc) {
                            const uint32_t slot = nc % kRingSlots, u = nc / kRingSlots;
                            ok = mbar_wait(&bars[kSBarFull + slot], u & 1u, abort_flag, kLimitNs);
                            if (!ok) break;
                            tc_fence_after();
#pragma unroll
                            for (int j = 0; j < kCopyChunks; ++j) {
                                const int c = kCopyChunks * k + j;  // chunk of the block
                                const uint64_t cd =
                                    ring_desc + (static_cast<uint64_t>(slot * kCopyBytes + j * kChunk) >> 4);
                                if (c < 8) {
                                    const uint32_t qa = tmem + kColQ + 32 * c;
                                    mma_ts(d, qa, cd, idesc, c ? 1u : 0u);
                                    mma_ts(d, qa + 8, cd + 2, idesc, 1u);
                                    mma_ts(d, qa + 16, cd + 4, idesc, 1u);
                                    mma_ts(d, qa + 24, cd + 6, idesc, 1u);
                                } else {
                                    mma_ss(d, qr_desc, cd, idesc, 1u);
                                    mma_ss(d, qr_desc + 2, cd + 2, idesc, 1u);
                                    mma_ss(d, qr_desc + 4, cd + 4, idesc, 1u);
                                    mma_ss(d, qr_desc + 6, cd + 6, idesc, 1u);
                                }
                            }
                            mma_commit(smem_u32(&bars[kSBarEmpty + slot]));
                        }
                        if (ok) mma_commit(smem_u32(&bars[kSBarSFull + sb]));
                    }
                }
                if (!ok) raise_abort(abort_flag, peer_abort, p.dev_status);
                mma_commit(smem_u32(&bars[kSBarFin]));
                mbar_wait(&bars[kSBarFin], 0, &never, kLimitNs);
            }
            __syncwarp();
        } else if (warp < kSoftWarps) {
            // ---- softmax: 8 warps; warp (q, hf) owns TMEM lanes 32q.. (query rows) and
            //      score columns 64hf .. 64hf + 63 of each 128-token tile
            const int qd = warp & 3, hf = warp >> 2;
            const int r = 32 * qd + lane;
            const uint32_t t_lane = tmem + (static_cast<uint32_t>(32 * qd) << 16);
            float* xchg = reinterpret_cast<float*>(smem + kSOffXchg);  // [2][128]
            const int rr = g * kRows + r;
            const bool row_ok = rr < p.R;
            const int j = row_ok ? rr / p.H : 0;
            SegWalk w, wn;
            w.init(wb0, wtb0, lo, hi, pidx);
            Seg s, sn;
            uint32_t n = 0;
            bool failed = false;
            bool have = w.next(p, s);
            while (!failed && have) {
                wn = w;
                const bool have_next = wn.next(p, sn);
                // this segment's absorbed query rows: latent part -> TMEM columns 0..255 (warp
                // hf=0: columns 0..127, hf=1: 128..255), RoPE part -> shared memory (hf=0: units
                // 0..3, hf=1: units 4..7).  The warp loads its 32 rows coalesced (a lane per
                // 16-byte unit) and transposes each 64-column chunk through a swizzled 4 KB tile
                // into the lane-per-row order of tcgen05.st.  The next segment's rows are pulled
                // into L2 two tiles before this segment ends (earlier, the streamed cache would
                // evict them).
                const int64_t qrow0 = static_cast<int64_t>(s.b) * p.R + g * kRows + 32 * qd;
                const int t_pf = max(s.t0, s.t1 - 2);
                const char* nq = (have_next && row_ok) ? reinterpret_cast<const char*>(
                                                              p.q + (static_cast<int64_t>(sn.b) * p.R + rr) * kRow)
                                                        : nullptr;
                {
                    uint8_t* qt = smem + kSOffQT + warp * (32 * 128);
                    const int lu = lane & 7, lr = lane >> 3;  // unit and row-in-quad of this lane's loads
#pragma unroll 1
                    for (int c = 4 * hf; c < 4 * hf + 4; c += 2) {
                        uint4 x[2][8];
#pragma unroll
                        for (int j = 0; j < 2; ++j)
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const int ri = 4 * i + lr;
                                x[j][i] = make_uint4(0, 0, 0, 0);
                                if (g * kRows + 32 * qd + ri < p.R)
                                    x[j][i] = reinterpret_cast<const uint4*>(p.q + (qrow0 + ri) * kRow)[8 * (c + j) + lu];
                            }
                        // the transpose tiles double as staging buffer 1: before the first write to them,
                        // wait until the sender has seen every copy of earlier messages read out
                        if (c == 4 * hf) bar_sync(kNbQFree, kSyncThreads);
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const int ri = 4 * i + lr;
                                *reinterpret_cast<uint4*>(qt + ri * 128 + ((lu ^ (ri & 7)) << 4)) = x[j][i];
                            }
                            __syncwarp();
                            uint32_t v[32];
#pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const uint4 y = *reinterpret_cast<const uint4*>(qt + lane * 128 + ((u ^ (lane & 7)) << 4));
                                v[4 * u] = y.x; v[4 * u + 1] = y.y; v[4 * u + 2] = y.z; v[4 * u + 3] = y.w;
                            }
                            __syncwarp();
                            tmem_st32(t_lane + kColQ + 32 * (c + j), v);
                        }
                    }
                    // RoPE part: rows 8 i + lane / 4, unit 4 hf + lane % 4, straight into its swizzled rows
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int ri = 8 * i + (lane >> 2), u = 4 * hf + (lane & 3);
                        uint4 y = make_uint4(0, 0, 0, 0);
                        if (g * kRows + 32 * qd + ri < p.R)
                            y = reinterpret_cast<const uint4*>(p.q + (qrow0 + ri) * kRow)[64 + u];
                        const int R = 32 * qd + ri;
                        *reinterpret_cast<uint4*>(smem + kSOffQR + R * 128 + ((u ^ (R & 7)) << 4)) = y;
                    }
                }
                fence_proxy_async_cta();
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars[kSBarQReady]);
                const int lim = row_ok ? (s.L - p.n_q + j + 1) : 0;  // keys 0 .. lim-1 are visible
                float m = -CUDART_INF_F, l = 0.f;
                for (int t = s.t0; t < s.t1; ++t, ++n) {
                    const uint32_t sb = n & 1u, us = n >> 1;
                    if (t == t_pf && have_next && row_ok)
                        for (int c = hf; c < 9; c += 2) prefetch_l2(nq + 128 * c);
                    bool ok = mbar_wait(&bars[kSBarSFull + sb], us & 1u, abort_flag, kLimitNs);
                    __syncwarp();
                    tc_fence_after();
                    float sv[64];
                    {
                        uint32_t a[32], b[32];
                        tmem_ld32(t_lane + col_s(sb) + 64 * hf, a);
                        tmem_ld32(t_lane + col_s(sb) + 64 * hf + 32, b);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            sv[k] = __uint_as_float(a[k]);
                            sv[32 + k] = __uint_as_float(b[k]);
                        }
                    }
                    tc_fence_before();
                    mbar_arrive(&bars[kSBarSEmpty + sb]);
                    const int nvalid = lim - t * kTile - 64 * hf;  // columns < nvalid are visible
                    if (nvalid < 64) {
#pragma unroll
                        for (int k = 0; k < 64; ++k) sv[k] = k < nvalid ? sv[k] : -CUDART_INF_F;
                    }
                    // row max over both halves (raw scores; the scale is positive)
                    xchg[hf * kRows + r] = fmax64(sv);
                    bar_sync(1 + qd, 64);
                    const float tmax = fmaxf(xchg[r], xchg[kRows + r]) * p.scale_log2;
                    const bool resc = tmax > m + kRescaleLog2;
                    float alpha = 1.f;
                    if (resc) {
                        alpha = (m == -CUDART_INF_F) ? 0.f : ex2_approx(m - tmax);
                        l *= alpha;
                        m = tmax;
                    }
                    const float mneg = (m == -CUDART_INF_F) ? 0.f : -m;
                    uint32_t pk[32];
                    float lsum = 0.f;
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        const float p0 = ex2_approx(fmaf(sv[2 * k], p.scale_log2, mneg));
                        const float p1 = ex2_approx(fmaf(sv[2 * k + 1], p.scale_log2, mneg));
                        lsum += p0 + p1;
                        pk[k] = cvt_bf16x2(p0, p1);
                    }
                    l += lsum;
                    if (bar_red_or(kNbFail, kSyncThreads, !ok || *abort_flag != 0)) {
                        failed = true;
                        break;
                    }
                    // the sender has seen the copy that last used this staging buffer (tile n - 2) read it
                    bar_sync(kNbStageFree, kSyncThreads);
                    uint8_t* stage = smem + ((n & 1u) ? kSOffStage1 : kSOffStage0);
                    uint8_t* prow = stage + hf * (kRows * 128) + r * 128;
                    // P row r, columns 64hf.. -> atom hf, row r: 16-byte units u at (u ^ (r % 8))
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        *reinterpret_cast<uint4*>(prow + ((u ^ (r & 7)) << 4)) =
                            make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                    if (hf == 0) reinterpret_cast<float*>(stage + kPBytes)[r] = alpha;
                    fence_proxy_async_cta();
                    bar_arrive(kNbStaged, kSyncThreads);
                }
                if (failed) break;
                // segment result: (m, l) with l summed over both column halves
                if (hf == 1) xchg[kRows + r] = l;
                bar_sync(1 + qd, 64);
                if (hf == 0 && row_ok)
                    p.ml_part[out_row_base + static_cast<int64_t>(s.slot) * kRows + r] = make_float2(m, l + xchg[kRows + r]);
                bar_sync(1 + qd, 64);
                w = wn;
                s = sn;
                have = have_next;
            }
            if (failed && tid == 0) raise_abort(abort_flag, peer_abort, p.dev_status);
        } else if (warp == kWarpSender) {
            // ---- sender: ships each staged P tile (one bulk copy, completing on the O CTA's
            //      barrier) once the O CTA has released that message slot.  Takes the same
            //      per-tile barrier steps as the softmax warps.
            const uint32_t peer_msg = mapa(sbase + kOOffMsg, peer);
            const uint32_t peer_pfull = mapa(sbase + kOOffBar + kOBarPFull * 8, peer);
            SegWalk w;
            w.init(wb0, wtb0, lo, hi, pidx);
            Seg s;
            uint32_t n = 0;
            bool failed = false;
            while (!failed && w.next(p, s)) {
                // every staged message read out before the Q reload reuses staging buffer 1
                if (lane == 0) bulk_wait_group_read<0>();
                __syncwarp();
                bar_arrive(kNbQFree, kSyncThreads);
                for (int t = s.t0; t < s.t1; ++t, ++n) {
                    const uint32_t pb = n % kPSlots, up = n / kPSlots;
                    if (bar_red_or(kNbFail, kSyncThreads, *abort_flag != 0)) {
                        failed = true;
                        break;
                    }
                    // the copy of tile n - 2 (same staging buffer as tile n) has read its source; the copy of
                    // tile n - 1 may still be queued
                    if (lane == 0) bulk_wait_group_read<1>();
                    __syncwarp();
                    bar_arrive(kNbStageFree, kSyncThreads);
                    bar_sync(kNbStaged, kSyncThreads);
                    if (lane == 0) {
                        if (mbar_wait<true>(&bars[kSBarPEmpty + pb], (up & 1u) ^ 1u, abort_flag, kLimitNs)) {
                            mbar_arrive_expect_tx_remote(peer_pfull + 8 * pb, kMsgBytes);
                            bulk_copy_to_peer(peer_msg + pb * kMsgStride,
                                              sbase + ((n & 1u) ? kSOffStage1 : kSOffStage0), kMsgBytes,
                                              peer_pfull + 8 * pb);
                            bulk_commit_group();
                        } else {
                            raise_abort(abort_flag, peer_abort, p.dev_status);
                        }
                    }
                    __syncwarp();
                }
            }
            if (lane == 0) bulk_wait_group_read<0>();
            __syncwarp();
        }
    } else if (active && rank == 1) {
        // =============================================================== O CTA
        if (warp == kWarpProducer) {
            // ---- copy producer: the 8 latent chunks of each block (its first 128 KB) = V,
            //      as four bulk copies of 2 chunks into the ring of V stages
            if (lane == 0) {
                SegWalk w;
                w.init(wb0, wtb0, lo, hi, pidx);
                Seg s;
                uint32_t nv = 0;  // stage loads issued
                bool ok = true;
                const uint64_t last_use = l2_policy_evict_first();
                while (ok && w.next(p, s)) {
                    for (int t = s.t0; ok && t < s.t1; ++t) {
                        const uint8_t* src = tile_src(p, s.tab[t]);
                        for (int k = 0; k < kVPerTile; ++k, ++nv) {
                            const uint32_t st = nv % kVStages, u = nv / kVStages;
                            if (!mbar_wait(&bars[kOBarVEmpty + st], (u & 1u) ^ 1u, abort_flag, kLimitNs)) {
                                ok = false;
                                break;
                            }
                            mbar_arrive_expect_tx(&bars[kOBarVFull + st], kVStageBytes);
                            bulk_load_hint(sbase + kOOffV + st * kVStageBytes, src + k * kVStageBytes, kVStageBytes,
                                           &bars[kOBarVFull + st], last_use);
                        }
                    }
                }
                if (!ok) raise_abort(abort_flag, peer_abort, p.dev_status);
                for (uint32_t i = (nv > kVStages ? nv - kVStages : 0); i < nv; ++i)
                    mbar_wait(&bars[kOBarVFull + i % kVStages], (i / kVStages) & 1u, &never, kLimitNs);
            }
        } else if (warp == kWarpMma) {
            // ---- MMA issuer (one thread): O += P V (A = P, K-major SW128; B = V, MN-major SW128
            //      with 16 KB between 64-column atoms)
            constexpr uint32_t idesc = idesc_bf16_f32(kRows, 64 * kVChunksPerStage, false, true);
            const uint32_t peer_pempty = mapa(sbase + kSOffBar + kSBarPEmpty * 8, peer);
            const uint64_t p_desc = sdesc_sw128(sbase + kOOffMsg, 16, 1024);
            const uint64_t v_desc = sdesc_sw128(sbase + kOOffV, kChunk, 1024);
            SegWalk w;
            w.init(wb0, wtb0, lo, hi, pidx);
            Seg s;
            uint32_t n = 0, nv = 0, kseg = 0, nresc = 0;
            bool ok = true;
            while (ok && w.next(p, s)) {
                for (int t = s.t0; ok && t < s.t1; ++t, ++n) {
                    const uint32_t pb = n % kPSlots, up = n / kPSlots;
                    const bool first = (t == s.t0);
                    if (lane == 0) {
                        ok = mbar_wait<true>(&bars[kOBarPFull + pb], up & 1u, abort_flag, kLimitNs);
                        if (ok && first) ok = mbar_wait(&bars[kOBarOFree], (kseg & 1u) ^ 1u, abort_flag, kLimitNs);
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    const uint8_t* msg = smem + kOOffMsg + pb * kMsgStride;
                    // some row's stale max moved iff its alpha is not exactly 1
                    const float4 al = reinterpret_cast<const float4*>(msg + kPBytes)[lane];
                    const bool resc = __any_sync(0xffffffffu, al.x != 1.f || al.y != 1.f || al.z != 1.f || al.w != 1.f);
                    if (!first && resc) {
                        // stale max moved: have the epilogue rescale O once all earlier MMAs are done
                        if (lane == 0) {
                            *resc_pb = static_cast<int>(pb);
                            mma_commit(smem_u32(&bars[kOBarODrain]));
                            mbar_arrive(&bars[kOBarRescReq]);
                            ok = mbar_wait(&bars[kOBarRescDone], nresc & 1u, abort_flag, kLimitNs);
                        }
                        ++nresc;
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                    }
                    const int nvalid = min(kTile, s.L - t * kTile);
                    for (int k = 0; k < kVPerTile; ++k, ++nv) {
                        const uint32_t st = nv % kVStages, u = nv / kVStages;
                        if (lane == 0) ok = mbar_wait(&bars[kOBarVFull + st], u & 1u, abort_flag, kLimitNs);
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                        constexpr int nch = kVChunksPerStage;
                        uint8_t* vst = smem + kOOffV + st * kVStageBytes;
                        if (nvalid < kTile) {
                            // rows past the sequence end: P is 0 there, make V 0 too (no 0 * NaN)
                            const int nz = (kTile - nvalid) * 8;  // 16-byte units per chunk
                            for (int i = lane; i < nch * nz; i += 32) {
                                const int c = i / nz, q = i % nz;
                                *reinterpret_cast<uint4*>(vst + c * kChunk + nvalid * 128 + q * 16) =
                                    make_uint4(0, 0, 0, 0);
                            }
                        }
                        // V may have been zeroed by this warp: order that before the tensor core reads
                        fence_proxy_async_cta();
                        __syncwarp();
                        if (lane == 0) {
                            tc_fence_after();
                            const uint64_t vd = v_desc + (static_cast<uint64_t>(st * kVStageBytes) >> 4);
                            const uint64_t pd = p_desc + (static_cast<uint64_t>(pb * kMsgStride) >> 4);
#pragma unroll
                            for (int kk = 0; kk < kTile / 16; ++kk)
                                mma_ss(tmem + 64 * kVChunksPerStage * k, pd + (((kk >> 2) * kRows * 128 + (kk & 3) * 32) >> 4),
                                       vd + ((kk * 2048) >> 4), idesc, (first && kk == 0) ? 0u : 1u);
                            mma_commit(smem_u32(&bars[kOBarVEmpty + st]));
                        }
                        __syncwarp();
                    }
                    if (!ok) break;
                    if (lane == 0) mma_commit(peer_pempty + 8 * pb);
                    __syncwarp();
                }
                if (!ok) break;
                if (lane == 0) mma_commit(smem_u32(&bars[kOBarOFull]));
                __syncwarp();
                ++kseg;
            }
            if (!ok && lane == 0) raise_abort(abort_flag, peer_abort, p.dev_status);
            if (lane == 0) {
                mma_commit(smem_u32(&bars[kOBarFin]));
                mbar_wait(&bars[kOBarFin], 0, &never, kLimitNs);
            }
            __syncwarp();
        } else if (warp < 4) {
            // ---- epilogue: warps 0..3, one thread per query row
            const int r = tid;
            const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
            SegWalk w;
            w.init(wb0, wtb0, lo, hi, pidx);
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
                        if (mbar_test(smem_u32(&bars[kOBarOFull]), kseg & 1u)) ev = 1;
                        else if (mbar_test(smem_u32(&bars[kOBarRescReq]), nresc & 1u)) ev = 2;
                        else if (*abort_flag) ev = 3;
                        else if ((++it & 255u) == 0 && globaltimer_ns() - t0 > kLimitNs) ev = 3;
                    }
                    ev = __shfl_sync(0xffffffffu, ev, 0);
                    if (ev == 1) {
                        ok = mbar_wait(&bars[kOBarOFull], kseg & 1u, abort_flag, kLimitNs);
                        break;
                    }
                    if (ev == 3) {
                        ok = false;
                        break;
                    }
                    if (ev == 2) {
                        ok = mbar_wait(&bars[kOBarRescReq], nresc & 1u, abort_flag, kLimitNs) &&
                             mbar_wait(&bars[kOBarODrain], nresc & 1u, abort_flag, kLimitNs);
                        __syncwarp();
                        tc_fence_after();
                        const float a =
                            reinterpret_cast<const float*>(smem + kOOffMsg + *resc_pb * kMsgStride + kPBytes)[r];
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
                        mbar_arrive(&bars[kOBarRescDone]);
                        ++nresc;
                        if (!__all_sync(0xffffffffu, ok)) {
                            ok = false;
                            break;
                        }
                        continue;
                    }
                    __nanosleep(256);
                }
                ok = __all_sync(0xffffffffu, ok);
                __syncwarp();
                if (!ok) break;
                tc_fence_after();
                // column group j (4 latent columns) of all 128 rows is contiguous, so each warp store
                // below writes 512 consecutive bytes (row-per-thread stores of row-major O would
                // scatter every warp store over 32 rows)
                float4* oseg = reinterpret_cast<float4*>(p.o_part) +
                               (out_row_base + static_cast<int64_t>(s.slot) * kRows) * (kDc / 4);
#pragma unroll 1
                for (int c = 0; c < 16; ++c) {
                    uint32_t v[32];
                    tmem_ld32(t_lane + 32 * c, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        oseg[(8 * c + k) * kRows + r] =
                            make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                        __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
                }
                tc_fence_before();
                mbar_arrive(&bars[kOBarOFree]);
                ++kseg;
            }
            if (!ok && lane == 0) raise_abort(abort_flag, peer_abort, p.dev_status);
        }
    }

    // ------------------------------------------------------------------ teardown
    grid_dependents_launch();  // the merge kernel may be scheduled; it waits for this grid to finish
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the peer no longer touches this CTA's shared memory
    if (warp == kWarpProducer) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace tc

// Co-resident clusters of the kernel on the current device, at most kMaxPairs (the workspace has a slot
// per pair).  The occupancy query runs once per device; the table is guarded for concurrent callers.
int decode_tc_clusters() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] > 0) return cache[dev];
    if (cudaFuncSetAttribute(tc::decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::kSmemBytes) !=
        cudaSuccess)
        return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * kMaxPairs);
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
    cache[dev] = n < kMaxPairs ? n : kMaxPairs;
    return cache[dev];
}

cudaError_t launch_decode_tc(const uint16_t* q, const uint8_t* cache, int64_t cap_blocks, const int32_t* block_table,
                             int max_blocks, const int32_t* kv_len, int B, int n_q, int H, float scale,
                             int clusters_per_group, float* o_part, float2* ml_part, int slots, int32_t* dev_status,
                             cudaStream_t stream) {
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
    tc::Params prm;
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
    prm.G = G;
    prm.P_g = P_g;
    prm.slots = slots;
    prm.scale_log2 = scale * 1.44269504088896340736f;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * G * P_g);
    cfg.blockDim = dim3(tc::kThreads);
    cfg.dynamicSmemBytes = tc::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, tc::decode_tc_kernel, prm);
}

}  // namespace mla
