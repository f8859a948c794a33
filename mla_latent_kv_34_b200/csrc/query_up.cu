// Query side of the low-rank path on tcgen05 tensor cores.
//
//   q^C[t, h, :] = W^UQ_h c^Q_t      (128 = [128 x d_c'] . d_c')
//   q^R[t, h, :] = W^QR_h c^Q_t      (64, not yet rotated; mla_absorb_q rotates it)
//
// The queries are compressed like the keys and values: a down-projection to c^Q
// and per-head up-projections from it (MLA explainer, 2.2.1.2: q^C_t = W^UQ c^Q_t;
// 2.2.2: the decoupled per-head query q^R).
//
// One CTA per (head, block of up to 128 tokens).  The contraction over d_c' is
// streamed through a ring of shared-memory stages, 64 columns per stage.  A
// stage holds the head's two weight slices stacked as one [192 x 64] chunk
// (W^UQ_h rows 0..127, W^QR_h rows 128..191) and the token slice [NT x 64], all
// loaded by TMA with the 128-byte swizzle.  Two M = 128 MMAs per K step use the
// chunk from row 0 (q^C into TMEM columns 0..127) and from row 64 (its lanes
// 64..127 are q^R, in TMEM columns 128..255), so no M = 64 accumulator layout is
// needed; the duplicated rows 64..127 of the second MMA are ignored.
//
// Warp roles: warps 0..3 read the accumulators back and store bf16; warp 4 lane 0
// issues the TMA loads; warp 5 lane 0 issues the MMAs.  Every wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "mla_internal.cuh"
#include "sm100.cuh"

namespace mla {
using namespace sm100;

namespace qup {

constexpr int kThreads = 192;
constexpr int kTokBlock = 128;                    // tokens per CTA (MMA N <= 128)
constexpr int kKChunk = 64;                       // d_c' columns per stage
constexpr int kUqBytes = 128 * kKChunk * 2;       // W^UQ_h slice, 16 KB
constexpr int kQrBytes = 64 * kKChunk * 2;        // W^QR_h slice, 8 KB
constexpr int kABytes = kUqBytes + kQrBytes;      // stacked [192 x 64] chunk
constexpr int kBBytes = kTokBlock * kKChunk * 2;  // token slice, up to 16 KB
constexpr int kStageBytes = kABytes + kBBytes;    // 40 KB
constexpr int kStages = 4;
constexpr int kOffBar = kStages * kStageBytes;
constexpr int kSmemBytes = kOffBar + 256;
constexpr int kTmemCols = 256;
constexpr uint64_t kLimitNs = 2000000000ull;
static_assert(kStageBytes % 1024 == 0 && kABytes % 1024 == 0, "swizzled TMA boxes need 1024-byte alignment");

__device__ __forceinline__ void tma_load_2d(uint32_t smem_dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__global__ void __launch_bounds__(kThreads, 1) query_up_kernel(
    const __grid_constant__ CUtensorMap uq_map, const __grid_constant__ CUtensorMap qr_map,
    const __grid_constant__ CUtensorMap cq_map, int T, int H, int d_cq, int NT, uint16_t* __restrict__ q_nope,
    uint16_t* __restrict__ q_rope, int32_t* dev_status) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);  // [kStages]
    uint64_t* empty = full + kStages;                               // [kStages]
    uint64_t* done = empty + kStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + 128);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffBar + 136);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x;
    const int t0 = blockIdx.y * kTokBlock;
    const int nt = min(kTokBlock, T - t0);
    const int KC = d_cq / kKChunk;
    if ((sbase & 1023u) != 0) {
        if (tid == 0) report(dev_status, MLA_DEVERR_TIMEOUT);
        return;
    }
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4 && lane == 0) {
        // producer: stage s of round n waits until the MMAs of round n-1 released it
        prefetch_tmap(&uq_map);
        prefetch_tmap(&qr_map);
        prefetch_tmap(&cq_map);
        const uint32_t tx = static_cast<uint32_t>(kABytes + NT * kKChunk * 2);
        for (int k = 0; k < KC; ++k) {
            const int s = k % kStages, n = k / kStages;
            if (n > 0 && !mbar_wait(&empty[s], (n - 1) & 1, abort_flag, kLimitNs)) {
                *abort_flag = 1;
                report(dev_status, MLA_DEVERR_TIMEOUT);
                break;
            }
            const uint32_t st = sbase + s * kStageBytes;
            mbar_arrive_expect_tx(&full[s], tx);
            tma_load_2d(st, &uq_map, k * kKChunk, h * 128, &full[s]);
            tma_load_2d(st + kUqBytes, &qr_map, k * kKChunk, h * 64, &full[s]);
            tma_load_2d(st + kABytes, &cq_map, k * kKChunk, t0, &full[s]);
        }
    } else if (warp == 5 && lane == 0) {
        // MMA issuer: D0 (cols 0..NT-1) = W^UQ_h c^Q, D1 (cols 128..) rows 64..191 of the stacked chunk
        const uint32_t idesc = idesc_bf16_f32(128, NT, false, false);
        for (int k = 0; k < KC; ++k) {
            const int s = k % kStages, n = k / kStages;
            if (!mbar_wait(&full[s], n & 1, abort_flag, kLimitNs)) {
                *abort_flag = 1;
                report(dev_status, MLA_DEVERR_TIMEOUT);
                break;
            }
            tc_fence_after();
            const uint32_t st = sbase + s * kStageBytes;
#pragma unroll
            for (int kk = 0; kk < kKChunk / 16; ++kk) {
                const uint64_t a0 = sdesc_sw128(st + kk * 32, 16, 1024);
                const uint64_t a1 = sdesc_sw128(st + 64 * 128 + kk * 32, 16, 1024);
                const uint64_t b = sdesc_sw128(st + kABytes + kk * 32, 16, 1024);
                const uint32_t acc = (k > 0 || kk > 0) ? 1u : 0u;
                mma_ss(tmem, a0, b, idesc, acc);
                mma_ss(tmem + 128, a1, b, idesc, acc);
            }
            mma_commit(smem_u32(&empty[s]));
        }
        mma_commit(smem_u32(done));  // fires once every MMA issued above has completed
    } else if (warp < 4) {
        // epilogue: lane 32w + l of D0 is q^C dim 32w + l; lanes 64..127 of D1 are q^R dims 0..63
        const bool ok = mbar_wait(done, 0, abort_flag, kLimitNs);
        __syncwarp();
        tc_fence_after();
        if (__all_sync(0xffffffffu, ok) && !*abort_flag) {
            const int d = 32 * warp + lane;
            for (int part = 0; part < (warp >= 2 ? 2 : 1); ++part) {
                const uint32_t col0 = part == 0 ? 0u : 128u;
                for (int j0 = 0; j0 < NT; j0 += 32) {
                    uint32_t v[32];
                    const uint32_t ta = tmem + (static_cast<uint32_t>(32 * warp) << 16) + col0 + j0;
                    if (NT - j0 >= 32) tmem_ld32(ta, v);
                    else tmem_ld16(ta, v);  // NT is a multiple of 16
                    tmem_wait_ld();
                    const int jn = min(32, nt - j0);
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (j < jn) {
                            const int64_t row = static_cast<int64_t>(t0 + j0 + j) * H + h;
                            const uint16_t y = f32_to_bf16_rne(__uint_as_float(v[j]));
                            if (part == 0) q_nope[row * kDh + d] = y;
                            else q_rope[row * kDr + (d - 64)] = y;
                        }
                    }
                }
            }
        } else if (lane == 0) {
            report(dev_status, MLA_DEVERR_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        // on an error path the epilogue may have left before the MMAs finished: their final
        // commit (always issued) must land before the columns are released
        volatile int never = 0;
        mbar_wait(done, 0, &never, kLimitNs);
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Row-major bf16 matrix [rows, cols] as a 2-D tensor map with [box_rows x 64] boxes, 128-byte swizzle.
bool matrix_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kKChunk), box_rows};
    cuuint32_t estr[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// MMA N (and token rows per TMA box) for T tokens: a multiple of 16, at most one token block.
int mma_n(int T) { return T >= kTokBlock ? kTokBlock : ((T + 15) & ~15); }

}  // namespace qup

cudaError_t launch_query_up(const uint16_t* c_q, const uint16_t* W_UQ, const uint16_t* W_QR, int T, int H, int d_cq,
                            uint16_t* q_nope, uint16_t* q_rope, int32_t* dev_status, cudaStream_t stream) {
    const int NT = qup::mma_n(T);
    CUtensorMap uq, qr, cq;
    if (!qup::matrix_map(&uq, W_UQ, static_cast<uint64_t>(H) * 128, d_cq, 128) ||
        !qup::matrix_map(&qr, W_QR, static_cast<uint64_t>(H) * 64, d_cq, 64) ||
        !qup::matrix_map(&cq, c_q, static_cast<uint64_t>(T), d_cq, static_cast<uint32_t>(NT)))
        return cudaErrorNotSupported;
    cudaError_t e =
        cudaFuncSetAttribute(qup::query_up_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, qup::kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(H, (T + qup::kTokBlock - 1) / qup::kTokBlock);
    qup::query_up_kernel<<<grid, qup::kThreads, qup::kSmemBytes, stream>>>(uq, qr, cq, T, H, d_cq, NT, q_nope, q_rope,
                                                                           dev_status);
    return cudaGetLastError();
}

}  // namespace mla
