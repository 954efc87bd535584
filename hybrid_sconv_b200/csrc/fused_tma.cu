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
// all completing on one mbarrier.  Tiles flow through a ring of STAGES
// shared-memory stages, so up to STAGES-1 tiles are in flight while one is
// computed: the memory system sees a steady stream of bulk copies whatever
// the register budget of the compute threads.  The grid is persistent, one
// block per resident slot (SMs x blocks per SM).  Work units are (token
// tile, channel block) pairs numbered token-tile major, u = tile * ncb + cb,
// and block b takes u = b, b + grid, b + 2 grid, ...: at any moment the grid
// works on one contiguous run of units, a compact band of x, out and the
// cache rows, and every block ends within one unit of the others.  DRAM
// serves that band far faster than one scattered spot per block (chunked
// prefill 82.2 -> 72.3 us, long prefill 611 -> 530 us, against equal
// contiguous shares of the units in channel-block-major order).  A block's
// channel block changes from unit to unit; it reloads its weights (a few
// lines, L1-resident) only when it does.
//
// Compute.  Eight warps per block; warp g owns tokens 4g..4g+3 of the tile
// and lane l the 16-byte pack of channels c0 + 8l .. c0 + 8l + 7.  Lanes
// 0..3 classify the warp's four tokens (ordinary, PAD, or needing cache
// taps / out of range) and compute their cache insert offsets once; when all
// four are ordinary -- nearly always in prefill -- one straight-line block
// convolves them from the W+3 shared-memory rows they need (16-byte loads,
// conflict-free: a warp reads one contiguous 512-byte row).  Otherwise each
// token takes the general path, where taps that precede the token's request
// come from the cache through the block table.  Outputs and cache inserts
// are 16-byte stores straight to global memory.
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
constexpr int kThreads = 256;      // 8 warps
constexpr int kTokPerWarp = kBT / (kThreads / 32);  // 4
constexpr int kMetaBytes = kBT * (8 + 8 + 4 + 4);   // positions, slots, seq_idx, query_start
constexpr uint32_t kWaitSpins = 1u << 22;  // bounded mbarrier polls (seconds, not forever)

template <int W>
struct Layout {
    static constexpr int rows = kBT + W - 1;
    static constexpr int x_bytes = rows * kBC * 2;  // multiple of 512: TMA destinations stay 128-B aligned
    static constexpr int stage = x_bytes + kMetaBytes;
};

template <int W, int STAGES>
constexpr int kStages_smem() {
    return STAGES * Layout<W>::stage + 2 * STAGES * 8;
}

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

// acc += w * tap for one 8-channel pack: eight fp32-accumulating FMAs that
// take bf16 operands directly (the product of two bf16 values is exact in
// fp32, so this equals widening both and one fmaf, bit for bit).  w holds
// the pack's weights for one lag as four bf16 pairs.
__device__ __forceinline__ void fma_pack(float (&acc)[8], const uint32_t (&w)[4], const P &tap) {
    const uint32_t q[4] = {tap.u.x, tap.u.y, tap.u.z, tap.u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        asm("{\n\t.reg .b16 wl, wh, tl, th;\n\t"
            "mov.b32 {wl, wh}, %2;\n\t"
            "mov.b32 {tl, th}, %3;\n\t"
            "fma.rn.f32.bf16 %0, wl, tl, %0;\n\t"
            "fma.rn.f32.bf16 %1, wh, th, %1;\n\t}"
            : "+f"(acc[2 * i]), "+f"(acc[2 * i + 1])
            : "r"(w[i]), "r"(q[i]));
}

// The pack's weights as bf16 pairs by lag (wb[d] multiplies position
// pos - d, weight column W-1-d); lags >= W are zero.
template <int W>
__device__ __forceinline__ void load_weights_bf16(const FusedArgs &a, int c, uint32_t (&wb)[4][4]) {
    const unsigned short *w = static_cast<const unsigned short *>(a.w);
    unsigned short e[8][4];
    if (a.w_vec) {  // dense [C, 4]: 32 contiguous elements
        union {
            uint4 u[4];
            unsigned short h[32];
        } raw;
        const uint4 *p = reinterpret_cast<const uint4 *>(w + static_cast<int64_t>(c) * 4);
#pragma unroll
        for (int q = 0; q < 4; ++q) raw.u[q] = __ldg(p + q);
#pragma unroll
        for (int v = 0; v < 8; ++v)
#pragma unroll
            for (int d = 0; d < 4; ++d) e[v][d] = raw.h[v * 4 + 3 - d];
    } else {
#pragma unroll
        for (int v = 0; v < 8; ++v)
#pragma unroll
            for (int d = 0; d < 4; ++d)
                e[v][d] = d < W ? __ldg(w + static_cast<int64_t>(c + v) * a.w_sc +
                                        static_cast<int64_t>(W - 1 - d) * a.w_sk)
                                : static_cast<unsigned short>(0);
    }
#pragma unroll
    for (int d = 0; d < 4; ++d)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            wb[d][i] = static_cast<uint32_t>(e[2 * i][d]) | (static_cast<uint32_t>(e[2 * i + 1][d]) << 16);
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// What a warp's lane u (< kTokPerWarp) knows about token u of its group.
enum : int { kSkip = 0, kFast = 1, kSlow = 2 };

template <int W, int STAGES, bool SILU, bool RESID>
__global__ void __launch_bounds__(kThreads, STAGES <= 3 ? 3 : 2)
fused_tma_kernel(const __grid_constant__ FusedArgs a, const __grid_constant__ TmaMaps maps) {
    using L = Layout<W>;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * L::stage);
    uint64_t *empty = full + STAGES;

    // This block's channel block and its token tiles g, g + G, ...
    // This block's units: u = b0, b0 + gstride, ... below ntiles * ncb.
    const int ntiles = (a.T + kBT - 1) / kBT;
    const int ncb = (a.C + kBC - 1) / kBC;
    const int64_t units = static_cast<int64_t>(ntiles) * ncb;
    const int64_t gstride = gridDim.x;
    const int64_t b0 = blockIdx.x;
    const int my = b0 < units ? static_cast<int>((units - 1 - b0) / gstride + 1) : 0;
    if (my <= 0) return;  // whole block

    if (threadIdx.x == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kThreads / 32);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    pdl_wait();  // inputs may come from the previous kernel in the stream
    pdl_trigger();

    int issued = 0;  // tiles issued so far (meaningful in thread 0, the producer)
    auto issue = [&](int k) {
        ++issued;
        const int s = k % STAGES;
        unsigned char *st = smem + s * L::stage;
        const int64_t u = b0 + k * gstride;
        const int c0 = static_cast<int>(u % ncb) * kBC;
        const int t0 = static_cast<int>(u / ncb) * kBT;
        mbar_expect_tx(&full[s], L::stage);
        tma_2d(st, &maps.x, c0, t0 - (W - 1), &full[s]);
        tma_1d(st + L::x_bytes, &maps.pos, t0, &full[s]);
        tma_1d(st + L::x_bytes + kBT * 8, &maps.slot, t0, &full[s]);
        tma_1d(st + L::x_bytes + kBT * 16, &maps.sid, t0, &full[s]);
        tma_1d(st + L::x_bytes + kBT * 20, &maps.qs, t0, &full[s]);
    };
    if (threadIdx.x == 0)
        for (int k = 0; k < STAGES && k < my; ++k) issue(k);

    const int lane_id = threadIdx.x & 31;
    const int i0 = (threadIdx.x >> 5) * kTokPerWarp;
    const int nv = a.C / 8;
    const int64_t slots_total = a.num_blocks * a.N;
    int cur_cb = -1;
    bool active = false;
    int c = 0;
    int64_t lane = 0;
    uint32_t wr[4][4];
    bool alive = true;
    int next = 0;  // the next tile this thread waits for

    for (int k = 0; k < my; ++k) {
        next = k;
        const int s = k % STAGES;
        const int64_t u = b0 + k * gstride;
        const int cb = static_cast<int>(u % ncb);
        const int t0 = static_cast<int>(u / ncb) * kBT;
        if (cb != cur_cb) {  // a new channel block: its taps and cache lanes
            cur_cb = cb;
            const int pack_raw = cb * (kBC / 8) + lane_id;
            active = pack_raw < nv;
            c = (active ? pack_raw : nv - 1) * 8;
            const int h = c / a.ws;
            lane = static_cast<int64_t>(h) * a.cs1 + a.off_s + (c - h * a.ws);
            load_weights_bf16<W>(a, c, wr);
        }
        if (!mbar_wait(&full[s], (k / STAGES) & 1)) {  // copies did not arrive in time
            if (a.err && lane_id == 0) atomicOr(a.err, static_cast<int>(SCONV_EFLAG_TIMEOUT));
            alive = false;
            break;
        }
        const unsigned char *st = smem + s * L::stage;
        const P *xs = reinterpret_cast<const P *>(st) + lane_id;  // row r at xs[r * 32]
        const int64_t *mpos = reinterpret_cast<const int64_t *>(st + L::x_bytes);
        const int64_t *mslot = mpos + kBT;
        const int32_t *msid = reinterpret_cast<const int32_t *>(st + L::x_bytes + kBT * 16);
        const int32_t *mqs = msid + kBT;

        // Lanes 0..3 classify the group's tokens and address their inserts.
        int code = kSkip;
        int64_t ins = 0;
        if (lane_id < kTokPerWarp) {
            const int i = i0 + lane_id;
            const int t = t0 + i;
            const int64_t slot = mslot[i];
            if (t < a.T && slot != -1) {
                const int64_t pos = mpos[i];
                const int req = msid[i];
                const int q0 = mqs[i];
                const bool bad = slot < 0 || slot >= slots_total || req < 0 ||
                                 req >= a.num_reqs || q0 < 0 || q0 > t || pos < 0;
                code = (!bad && t - q0 >= W - 1) ? kFast : kSlow;
                if (!bad) {
                    int64_t blk, off;
                    split_n(a, slot, a.slots32 != 0, blk, off);
                    ins = blk * a.cs0 + off * a.cs2;
                }
            }
        }
        const unsigned fast_mask = __ballot_sync(0xffffffffu, code == kFast);

        // Shared-memory row r holds x row t0 - (W-1) + r; token i at lag d
        // reads row i + (W-1) - d.
        P rows[kTokPerWarp + W - 1];
#pragma unroll
        for (int r = 0; r < kTokPerWarp + W - 1; ++r) rows[r] = xs[(i0 + r) * 32];

        bf16 *out = static_cast<bf16 *>(a.out);
        bf16 *cache = static_cast<bf16 *>(a.cache);
        if ((fast_mask & 0xfu) == 0xfu) {
            // The common case: four ordinary tokens, straight-line code.
#pragma unroll
            for (int uu = 0; uu < kTokPerWarp; ++uu) {
                float acc[8];
#pragma unroll
                for (int v = 0; v < 8; ++v) acc[v] = 0.f;
#pragma unroll
                for (int d = W - 1; d >= 0; --d) fma_pack(acc, wr[d], rows[uu + W - 1 - d]);
                const int64_t ins_u = __shfl_sync(0xffffffffu, ins, uu);
                float xc[8];
                rows[uu + W - 1].to_float(xc);
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    float y = acc[v];
                    if (SILU) y = silu<bf16>(y);
                    if (RESID) y = __fadd_rn(y, xc[v]);  // never contracted into an FMA
                    acc[v] = y;
                }
                P o;
                o.from_float(acc);
                if (active) {
                    o.store(out + static_cast<int64_t>(t0 + i0 + uu) * a.out_rs + c);
                    rows[uu + W - 1].store(cache + ins_u + lane);
                }
            }
        } else {
#pragma unroll
            for (int uu = 0; uu < kTokPerWarp; ++uu) {
                const int code_u = __shfl_sync(0xffffffffu, code, uu);
                const int64_t ins_u = __shfl_sync(0xffffffffu, ins, uu);
                if (code_u == kSkip) continue;  // PAD row or past T
                const int i = i0 + uu;
                const int t = t0 + i;
                float acc[8];
#pragma unroll
                for (int v = 0; v < 8; ++v) acc[v] = 0.f;
                if (code_u == kFast) {
#pragma unroll
                    for (int d = W - 1; d >= 0; --d) fma_pack(acc, wr[d], rows[uu + W - 1 - d]);
                } else {
                    // Taps before the request's first row come from the cache
                    // (zero before position 0), or an index is out of range.
                    const int64_t slot = mslot[i];
                    const int64_t pos = mpos[i];
                    const int req = msid[i];
                    const int q0 = mqs[i];
                    unsigned bad = 0;
                    if (slot < 0 || slot >= slots_total) bad |= SCONV_EFLAG_SLOT;
                    if (req < 0 || req >= a.num_reqs) bad |= SCONV_EFLAG_REQUEST;
                    if (q0 < 0 || q0 > t) bad |= SCONV_EFLAG_QUERY_START;
                    if (pos < 0) bad |= SCONV_EFLAG_POSITION;
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
                            fma_pack(acc, wr[d], rows[uu + W - 1 - d]);
                        else if (pos - d >= 0)
                            fma_pack(acc, wr[d], ct[d]);
                    }
                }
                float xc[8];
                rows[uu + W - 1].to_float(xc);
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    float y = acc[v];
                    if (SILU) y = silu<bf16>(y);
                    if (RESID) y = __fadd_rn(y, xc[v]);  // never contracted into an FMA
                    acc[v] = y;
                }
                P o;
                o.from_float(acc);
                if (active) {
                    o.store(out + static_cast<int64_t>(t) * a.out_rs + c);
                    rows[uu + W - 1].store(cache + ins_u + lane);
                }
            }
        }
        // This warp is done with stage s.  The producer refills the stage
        // of the previous tile once all eight warps have released it, so a
        // warp never waits for the others to finish the tile it is on.
        __syncwarp();
        if (lane_id == 0) mbar_arrive(&empty[s]);
        next = k + 1;
        if (threadIdx.x == 0 && k >= 1 && k - 1 + STAGES < my) {
            const int j = k - 1;
            if (mbar_wait(&empty[j % STAGES], (j / STAGES) & 1)) {
                issue(j + STAGES);
            } else {
                if (a.err) atomicOr(a.err, static_cast<int>(SCONV_EFLAG_TIMEOUT));
                alive = false;
                break;
            }
        }
    }
    if (!alive && threadIdx.x == 0) {
        // Let the copies this block issued and has not consumed land before
        // its shared memory is released (each wait bounded).
        for (int j = next; j < issued; ++j) mbar_wait(&full[j % STAGES], (j / STAGES) & 1);
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

constexpr int kLaunchStages = 4;

template <int W, bool SILU, bool RESID>
cudaError_t launch_flags(const FusedArgs &a, const TmaMaps &maps, cudaStream_t stream) {
    constexpr int S = kLaunchStages;
    constexpr int smem = kStages_smem<W, S>();
    auto kernel = fused_tma_kernel<W, S, SILU, RESID>;
    // Resident blocks per SM and the SM count, once per process and kernel
    // (the grid is a function of the device and of T and C only).
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    static int per_sm = 1, sms = 148;
    std::call_once(once, [&] {
        attr = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (attr != cudaSuccess) return;
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem) !=
                cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
    });
    if (attr != cudaSuccess) return attr;
    // One block per resident slot, at most one per unit.
    const int64_t ntiles = (a.T + kBT - 1) / kBT;
    const int64_t ncb = (a.C + kBC - 1) / kBC;
    int64_t grid = static_cast<int64_t>(sms) * per_sm;
    if (grid > ntiles * ncb) grid = ntiles * ncb;
    return launch_pdl(kernel, dim3(static_cast<unsigned>(grid)), dim3(kThreads), smem, stream,
                      a, maps);
}

template <int W>
cudaError_t launch_w(const FusedArgs &a, const TmaMaps &maps, cudaStream_t stream) {
    if (a.silu) {
        return a.resid ? launch_flags<W, true, true>(a, maps, stream)
                       : launch_flags<W, true, false>(a, maps, stream);
    }
    return a.resid ? launch_flags<W, false, true>(a, maps, stream)
                   : launch_flags<W, false, false>(a, maps, stream);
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
