// fused_tma.cu -- the prefill form of the fused insert + causal conv1d
// ("vllm.models.inkling.nvidia.ops.sconv", fused_sconv) with its x tiles
// and per-token metadata staged in shared memory by the Tensor Memory
// Accelerator, for sm_100a.
//
// Tiling.  A tile is kBT = 32 consecutive tokens x kBC = 256 channels
// (512 bytes of bf16 per row).  One thread of each block issues, per tile,
//   * a 2-D tensor copy of x rows [t0 - (W-1), t0 + 32) x [c0, c0 + 256)
//     (the W-1 halo rows before the tile included; rows before 0 and past T
//     and channels past C arrive as zeros), and
//   * four 1-D tensor copies of the tile's positions, slot_mapping, seq_idx
//     and query_start,
// all completing on one mbarrier.  Tiles flow through a kStages-deep ring of
// shared-memory stages, so up to kStages-1 tiles are in flight while one is
// computed: the memory system sees a steady stream of bulk copies whatever
// the register budget of the compute threads.
//
// Compute.  Eight warps per block; warp g owns tokens 4g..4g+3 of the tile
// and lane l the 16-byte pack of channels c0 + 8l .. c0 + 8l + 7.  A thread
// reads the W+3 rows its four tokens need once from shared memory (16-byte
// loads, conflict-free: a warp reads one contiguous 512-byte row), and per
// token convolves, applies the epilogue and stores its output pack and its
// cache insert straight to global memory.  Taps that precede the token's
// request come from the cache through the block table (the first W-1
// tokens of each request only).
//
// Every wait on an mbarrier is bounded; a block whose copies do not arrive
// in time sets SCONV_EFLAG_TIMEOUT, waits (bounded) for its other copies and
// returns without writing anything for that tile.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "fused_common.cuh"
#include "sconv.h"

namespace sconv {
namespace {

constexpr int kBC = 256;           // channels per tile
constexpr int kBT = 32;            // tokens per tile
constexpr int kStages = 4;         // shared-memory ring depth
constexpr int kThreads = 256;      // 8 warps
constexpr int kTokPerWarp = kBT / (kThreads / 32);  // 4
constexpr int kMetaBytes = kBT * (8 + 8 + 4 + 4);   // positions, slots, seq_idx, query_start
constexpr uint32_t kWaitSpins = 1u << 22;  // bounded mbarrier polls (seconds, not forever)

template <int W>
struct Layout {
    static constexpr int rows = kBT + W - 1;
    static constexpr int x_bytes = rows * kBC * 2;  // multiple of 512: TMA destinations stay 128-B aligned
    static constexpr int stage = x_bytes + kMetaBytes;
    static constexpr int smem = kStages * stage + kStages * 8;
};

struct TmaMaps {
    CUtensorMap x, pos, slot, sid, qs;
};

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait for the phase with the given parity to complete.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitSpins; ++i)
        if (mbar_test(bar, parity)) return true;
    return false;
}

__device__ __forceinline__ void tma_2d(void *dst, const CUtensorMap *map, int x, int y,
                                       uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tma_1d(void *dst, const CUtensorMap *map, int x, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.1d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2}], [%3];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(smem_addr(bar))
        : "memory");
}

using P = Pack<bf16, 8>;

// acc += w * tap for one 8-channel pack, as four packed fp32 FMAs.
__device__ __forceinline__ void fma_pack(float (&acc)[8], const float (&w)[8], const P &tap) {
    const uint32_t q[4] = {tap.u.x, tap.u.y, tap.u.z, tap.u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        fma2(acc[2 * i], acc[2 * i + 1], w[2 * i], w[2 * i + 1], __uint_as_float(q[i] << 16),
             __uint_as_float(q[i] & 0xffff0000u));
}

template <int W>
__global__ void __launch_bounds__(kThreads, 2)
fused_tma_kernel(const __grid_constant__ FusedArgs a, const __grid_constant__ TmaMaps maps,
                 int tiles_per_block) {
    using L = Layout<W>;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * L::stage);

    const int ntiles = (a.T + kBT - 1) / kBT;
    const int tile0 = blockIdx.x * tiles_per_block;
    const int my = min(tiles_per_block, ntiles - tile0);
    if (my <= 0) return;  // whole block
    const int c0 = blockIdx.y * kBC;

    if (threadIdx.x == 0) {
#pragma unroll
        for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    pdl_wait();  // inputs may come from the previous kernel in the stream
    pdl_trigger();

    auto issue = [&](int k) {
        const int s = k % kStages;
        unsigned char *st = smem + s * L::stage;
        const int t0 = (tile0 + k) * kBT;
        mbar_expect_tx(&full[s], L::stage);
        tma_2d(st, &maps.x, c0, t0 - (W - 1), &full[s]);
        tma_1d(st + L::x_bytes, &maps.pos, t0, &full[s]);
        tma_1d(st + L::x_bytes + kBT * 8, &maps.slot, t0, &full[s]);
        tma_1d(st + L::x_bytes + kBT * 16, &maps.sid, t0, &full[s]);
        tma_1d(st + L::x_bytes + kBT * 20, &maps.qs, t0, &full[s]);
    };
    if (threadIdx.x == 0)
        for (int k = 0; k < kStages && k < my; ++k) issue(k);

    const int lane_id = threadIdx.x & 31;
    const int grp = threadIdx.x >> 5;
    const int nv = a.C / 8;
    const int pack_raw = c0 / 8 + lane_id;
    const bool active = pack_raw < nv;
    const int c = (active ? pack_raw : nv - 1) * 8;
    const int h = c / a.ws;
    const int64_t lane = static_cast<int64_t>(h) * a.cs1 + a.off_s + (c - h * a.ws);
    float wr[4][8];
    load_weights<bf16, 8, 4>(a, c, wr);

    for (int k = 0; k < my; ++k) {
        const int s = k % kStages;
        const bool ok = mbar_wait(&full[s], (k / kStages) & 1);
        if (__syncthreads_or(!ok)) {
            // Copies did not arrive: report, let the others land, stop.
            if (threadIdx.x == 0) {
                if (a.err) atomicOr(a.err, static_cast<int>(SCONV_EFLAG_TIMEOUT));
                for (int j = k; j < my && j < k + kStages; ++j)
                    mbar_wait(&full[j % kStages], (j / kStages) & 1);
            }
            __syncthreads();
            return;
        }
        const unsigned char *st = smem + s * L::stage;
        const P *xs = reinterpret_cast<const P *>(st) + lane_id;  // row r at xs[r * 32]
        const int64_t *mpos = reinterpret_cast<const int64_t *>(st + L::x_bytes);
        const int64_t *mslot = mpos + kBT;
        const int32_t *msid = reinterpret_cast<const int32_t *>(st + L::x_bytes + kBT * 16);
        const int32_t *mqs = msid + kBT;
        const int t0 = (tile0 + k) * kBT;
        const int i0 = grp * kTokPerWarp;

        // Shared-memory row r holds x row t0 - (W-1) + r; token i at lag d
        // reads row i + (W-1) - d.
        P rows[kTokPerWarp + W - 1];
#pragma unroll
        for (int r = 0; r < kTokPerWarp + W - 1; ++r) rows[r] = xs[(i0 + r) * 32];

#pragma unroll
        for (int u = 0; u < kTokPerWarp; ++u) {
            const int i = i0 + u;
            const int t = t0 + i;
            if (t >= a.T) break;
            const int64_t slot = mslot[i];
            if (slot == -1) continue;  // PAD row
            const int64_t pos = mpos[i];
            const int req = msid[i];
            const int q0 = mqs[i];
            unsigned bad = 0;
            if (slot < 0 || slot >= a.num_blocks * a.N) bad |= SCONV_EFLAG_SLOT;
            if (req < 0 || req >= a.num_reqs) bad |= SCONV_EFLAG_REQUEST;
            if (q0 < 0 || q0 > t) bad |= SCONV_EFLAG_QUERY_START;
            if (pos < 0) bad |= SCONV_EFLAG_POSITION;

            float acc[8];
#pragma unroll
            for (int v = 0; v < 8; ++v) acc[v] = 0.f;
            if (!bad && t - q0 >= W - 1) {
                // Every tap is an x row of this step, in shared memory.
#pragma unroll
                for (int d = W - 1; d >= 0; --d) fma_pack(acc, wr[d], rows[u + W - 1 - d]);
            } else {
                // First W-1 tokens of a request: earlier taps from the cache
                // (zero before position 0).
                P ct[W];
#pragma unroll
                for (int d = 1; d < W; ++d)
                    if (t - d < q0 && pos - d >= 0 && !bad)
                        bad |= load_cache_tap<bf16, 8>(a, req, pos - d, lane, ct[d]);
                if (bad) {
                    if (a.err && active) atomicOr(a.err, static_cast<int>(bad));
                    continue;
                }
#pragma unroll
                for (int d = W - 1; d >= 0; --d) {
                    if (d == 0 || t - d >= q0)
                        fma_pack(acc, wr[d], rows[u + W - 1 - d]);
                    else if (pos - d >= 0)
                        fma_pack(acc, wr[d], ct[d]);
                }
            }
            if (!active) continue;
            float xc[8];
            rows[u + W - 1].to_float(xc);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                float y = acc[v];
                if (a.silu) y = silu<bf16>(y);
                if (a.resid) y += xc[v];
                acc[v] = y;
            }
            P o;
            o.from_float(acc);
            o.store(static_cast<bf16 *>(a.out) + static_cast<int64_t>(t) * a.out_rs + c);
            int64_t blk, off;
            split_n(a, slot, a.slots32 != 0, blk, off);
            rows[u + W - 1].store(static_cast<bf16 *>(a.cache) + blk * a.cs0 + off * a.cs2 + lane);
        }
        __syncthreads();  // every warp is done with stage s
        if (threadIdx.x == 0 && k + kStages < my) issue(k + kStages);
    }
}

// cuTensorMapEncodeTiled, fetched from the driver once (no link to libcuda).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool encode_1d(CUtensorMap *m, CUtensorMapDataType type, const void *base, int64_t n) {
    const cuuint64_t dim[1] = {static_cast<cuuint64_t>(n)};
    const cuuint32_t box[1] = {kBT};
    const cuuint32_t elem[1] = {1};
    const cuuint64_t no_strides[1] = {0};  // rank 1 has no strides, but the array must exist
    return encode_fn()(m, type, 1, const_cast<void *>(base), dim, no_strides, box, elem,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_NONE,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int W>
cudaError_t launch_w(const FusedArgs &a, const TmaMaps &maps, cudaStream_t stream) {
    using L = Layout<W>;
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    std::call_once(once, [] {
        attr = cudaFuncSetAttribute(fused_tma_kernel<W>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, L::smem);
    });
    if (attr != cudaSuccess) return attr;
    const int ntiles = (a.T + kBT - 1) / kBT;
    const int cblocks = (a.C + kBC - 1) / kBC;
    // About three resident blocks per SM across the grid, each streaming a
    // run of consecutive tiles of one channel block.
    const int64_t target = 148LL * 3;
    int per = static_cast<int>((static_cast<int64_t>(ntiles) * cblocks + target - 1) / target);
    if (per < 1) per = 1;
    const dim3 grid((ntiles + per - 1) / per, cblocks);
    return launch_pdl(fused_tma_kernel<W>, grid, dim3(kThreads), L::smem, stream, a, maps, per);
}

}  // namespace

cudaError_t launch_fused_tma(const FusedArgs &a, cudaStream_t stream, bool &used) {
    used = false;
    auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (a.W < 1 || a.W > 4 || a.C < kBC || encode_fn() == nullptr) return cudaSuccess;
    if (!al16(a.x) || (a.x_rs * 2) % 16 != 0 || !al16(a.positions) || !al16(a.slot) ||
        !al16(a.seq_idx) || !al16(a.qstart))
        return cudaSuccess;
    TmaMaps maps;
    {
        const cuuint64_t dim[2] = {static_cast<cuuint64_t>(a.C), static_cast<cuuint64_t>(a.T)};
        const cuuint64_t stride[1] = {static_cast<cuuint64_t>(a.x_rs) * 2};
        const cuuint32_t box[2] = {kBC, static_cast<cuuint32_t>(kBT + a.W - 1)};
        const cuuint32_t elem[2] = {1, 1};
        if (encode_fn()(&maps.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(a.x), dim,
                        stride, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaSuccess;
    }
    if (!encode_1d(&maps.pos, CU_TENSOR_MAP_DATA_TYPE_INT64, a.positions, a.T) ||
        !encode_1d(&maps.slot, CU_TENSOR_MAP_DATA_TYPE_INT64, a.slot, a.T) ||
        !encode_1d(&maps.sid, CU_TENSOR_MAP_DATA_TYPE_INT32, a.seq_idx, a.T) ||
        !encode_1d(&maps.qs, CU_TENSOR_MAP_DATA_TYPE_INT32, a.qstart, a.T))
        return cudaSuccess;
    used = true;
    switch (a.W) {
        case 1: return launch_w<1>(a, maps, stream);
        case 2: return launch_w<2>(a, maps, stream);
        case 3: return launch_w<3>(a, maps, stream);
        default: return launch_w<4>(a, maps, stream);
    }
}

}  // namespace sconv
