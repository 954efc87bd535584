// gather.cu -- prefix-caching snapshots beyond the dense conv windows, sm_100a:
//
//  * scatter_ssm_* -- conditional gather of SSM chunk-scan state rows
//    ("core.ssm.ops.intermediate_extraction", _scatter_intermediate_ssm_kernel
//    / scatter_intermediate_ssm): out row i = states row chunk_indices[i] for
//    slots i < *real_count.  Grid (row blocks, max_count): sized from
//    max_count and the row length only; every block reads the device count
//    and returns at once when its slot is beyond it, so padded slots move no
//    data.  Each thread copies kUnroll 16-byte chunks (independent loads in
//    flight), or single elements when a row is not 16-byte aligned.
//  * extract_paged_* -- the length-d_conv window gather of
//    sconv_extract_windows with the conv input read from the paged cache of
//    "vllm.models.inkling.nvidia.ops.sconv" through the block table: a
//    thread loads the d_conv 16-byte cache rows of one channel pack and
//    stores them transposed (out[slot][c][k], k contiguous).
//
// A slot whose index is out of range writes nothing and reports through the
// optional error flag; nothing traps or waits.
#include "common.cuh"
#include "sconv.h"

namespace sconv {
namespace {

constexpr int kUnroll = 4;

__device__ __forceinline__ int clamp_count(const int32_t *real_count, int max_count) {
    int rc = __ldg(real_count);
    if (rc < 0) rc = 0;
    if (rc > max_count) rc = max_count;
    return rc;
}

// 16-byte chunks: row lengths, strides and bases all 16-byte aligned.
__global__ void __launch_bounds__(256) scatter_ssm_vec(const __grid_constant__ SsmArgs a,
                                                       int64_t chunks_per_row,
                                                       int64_t states_rs16, int64_t out_rs16) {
    const int slot = blockIdx.y;
    if (threadIdx.x == 0) {
        prefetch_l2(a.real_count);
        prefetch_l2(a.idx + slot);
    }
    pdl_wait();
    pdl_trigger();
    if (slot >= clamp_count(a.real_count, a.max_count)) return;
    const int64_t row = __ldg(a.idx + slot);
    if (row < 0 || row >= a.num_chunks) {
        if (a.err && threadIdx.x == 0 && blockIdx.x == 0)
            atomicOr(a.err, static_cast<int>(SCONV_EFLAG_REQUEST));
        return;
    }
    const uint4 *src = static_cast<const uint4 *>(a.states) + row * states_rs16;
    uint4 *dst = static_cast<uint4 *>(a.out) + static_cast<int64_t>(slot) * out_rs16;
    const int64_t base = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * kUnroll;
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
        if (base + u < chunks_per_row) v[u] = __ldg(src + base + u);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
        if (base + u < chunks_per_row) dst[base + u] = v[u];
}

// Any alignment: one element (R = 2- or 4-byte raw type) per thread.
template <typename R>
__global__ void __launch_bounds__(256) scatter_ssm_elem(const __grid_constant__ SsmArgs a) {
    const int slot = blockIdx.y;
    pdl_wait();
    pdl_trigger();
    if (slot >= clamp_count(a.real_count, a.max_count)) return;
    const int64_t row = __ldg(a.idx + slot);
    if (row < 0 || row >= a.num_chunks) {
        if (a.err && threadIdx.x == 0 && blockIdx.x == 0)
            atomicOr(a.err, static_cast<int>(SCONV_EFLAG_REQUEST));
        return;
    }
    const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e >= a.state_flat) return;
    static_cast<R *>(a.out)[static_cast<int64_t>(slot) * a.out_rs + e] =
        __ldg(static_cast<const R *>(a.states) + row * a.states_rs + e);
}

// Resolve slot i's window: the physical block of each tap position (-1 for
// p < 0).  Returns the SCONV_EFLAG_* bits of an out-of-range index, else 0.
// r and end are the slot's request and end position, loaded by the caller.
template <int DC>
__device__ __forceinline__ unsigned window_blocks(const PagedExtractArgs &a, int r, int64_t end,
                                                  int d_conv, int64_t (&blk)[DC > 0 ? DC : 8],
                                                  int64_t (&off)[DC > 0 ? DC : 8]) {
    if (r < 0 || r >= a.num_reqs) return SCONV_EFLAG_REQUEST;
    const int32_t *bt_row = a.bt + static_cast<int64_t>(r) * a.bt_rs;
    // One division per slot: (lb, o) = the block and offset of the first
    // non-negative tap position, then stepped along the window.
    const int64_t p0 = end - d_conv;
    int64_t lb = (p0 < 0 ? 0 : p0) / a.N;
    int64_t o = (p0 < 0 ? 0 : p0) - lb * a.N;
    int64_t loaded = -1;
    int32_t b = -1;
#pragma unroll
    for (int k = 0; k < (DC > 0 ? DC : 8); ++k) {
        blk[k] = -1;
        if (k >= d_conv) continue;
        if (p0 + k < 0) continue;
        if (lb >= a.max_blocks) return SCONV_EFLAG_LOGICAL;
        if (lb != loaded) {
            b = __ldg(bt_row + lb);
            loaded = lb;
            if (b < 0 || b >= a.num_blocks) return SCONV_EFLAG_BLOCK;
        }
        blk[k] = b;
        off[k] = o;
        if (++o == a.N) {
            o = 0;
            ++lb;
        }
    }
    return 0;
}

// 16-byte channel packs (VEC elements of raw type R), DC taps per window.
// Before the PDL wait the thread resolves its window *speculatively*
// (L2-only loads of real_count, the slot's request and end position and
// the block-table entries, each range-checked) and prefetches the cache rows
// into L2; after the wait the same chain runs with ordinary loads, now L2
// hits.  real_count, the request and the end position are loaded together.
template <typename R, int DC>
__global__ void __launch_bounds__(256) extract_paged_vec(const __grid_constant__ PagedExtractArgs a) {
    constexpr int VEC = 16 / sizeof(R);
    const int slot = blockIdx.x;
    const int pack = blockIdx.y * blockDim.x + threadIdx.x;
    const bool in_range = pack < a.H * a.ws / VEC;
    const int c = pack * VEC;
    const int h = c / a.ws;
    const int64_t lane = static_cast<int64_t>(h) * a.cs1 + a.off_s + (c - h * a.ws);
    const R *cache = static_cast<const R *>(a.cache);
    if (in_range && slot < __ldcg(a.real_count)) {
        const int r = __ldcg(a.request + slot);
        const int64_t end = __ldcg(a.abs_pos + slot);
        if (r >= 0 && r < a.num_reqs) {
            const int32_t *bt_row = a.bt + static_cast<int64_t>(r) * a.bt_rs;
#pragma unroll
            for (int k = 0; k < DC; ++k) {
                const int64_t p = end - DC + k;
                if (p < 0) continue;
                const int64_t lb = p / a.N;
                if (lb >= a.max_blocks) break;
                const int32_t b = __ldcg(bt_row + lb);
                if (b < 0 || b >= a.num_blocks) break;
                prefetch_l2(cache + b * a.cs0 + (p - lb * a.N) * a.cs2 + lane);
            }
        }
    }
    pdl_wait();
    pdl_trigger();
    const int rc = clamp_count(a.real_count, a.max_count);
    const int r = __ldg(a.request + slot);  // slot < max_count: always in bounds
    const int64_t end = __ldg(a.abs_pos + slot);
    if (slot >= rc) return;
    int64_t blk[DC], off[DC];
    const unsigned bad = window_blocks<DC>(a, r, end, DC, blk, off);
    if (bad) {
        if (a.err && threadIdx.x == 0 && blockIdx.y == 0) atomicOr(a.err, static_cast<int>(bad));
        return;
    }
    if (!in_range) return;
    union U {
        uint4 u;
        R e[VEC];
    };
    U rows[DC];
#pragma unroll
    for (int k = 0; k < DC; ++k) {
        if (blk[k] >= 0)
            rows[k].u = __ldg(reinterpret_cast<const uint4 *>(cache + blk[k] * a.cs0 +
                                                              off[k] * a.cs2 + lane));
        else
            rows[k].u = make_uint4(0u, 0u, 0u, 0u);
    }
    U outv[DC];
#pragma unroll
    for (int v = 0; v < VEC; ++v)
#pragma unroll
        for (int k = 0; k < DC; ++k) {
            const int flat = v * DC + k;
            outv[flat / VEC].e[flat % VEC] = rows[k].e[v];
        }
    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<R *>(a.out) + slot * a.out_ss +
                                           static_cast<int64_t>(c) * DC);
#pragma unroll
    for (int q = 0; q < DC; ++q) dst[q] = outv[q].u;
}

// Any layout: one channel per thread, element copies.
template <typename R>
__global__ void __launch_bounds__(256) extract_paged_elem(const __grid_constant__ PagedExtractArgs a) {
    const int slot = blockIdx.x;
    pdl_wait();
    pdl_trigger();
    if (slot >= clamp_count(a.real_count, a.max_count)) return;
    int64_t blk[8], off[8];
    const unsigned bad = window_blocks<0>(a, __ldg(a.request + slot), __ldg(a.abs_pos + slot),
                                          a.d_conv, blk, off);
    if (bad) {
        if (a.err && threadIdx.x == 0 && blockIdx.y == 0) atomicOr(a.err, static_cast<int>(bad));
        return;
    }
    const int c = blockIdx.y * blockDim.x + threadIdx.x;
    if (c >= a.H * a.ws) return;
    const int h = c / a.ws;
    const int64_t lane = static_cast<int64_t>(h) * a.cs1 + a.off_s + (c - h * a.ws);
    const R *cache = static_cast<const R *>(a.cache);
    R *dst = static_cast<R *>(a.out) + slot * a.out_ss + static_cast<int64_t>(c) * a.d_conv;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (k >= a.d_conv) break;
        dst[k] = blk[k] >= 0 ? __ldg(cache + blk[k] * a.cs0 + off[k] * a.cs2 + lane) : R(0);
    }
}

template <typename R>
cudaError_t launch_paged_t(const PagedExtractArgs &a, bool vec, cudaStream_t stream) {
    const int C = a.H * a.ws;
    if (!vec) {
        const int threads = C >= 256 ? 256 : 64;
        return launch_pdl(extract_paged_elem<R>, dim3(a.max_count, (C + threads - 1) / threads),
                          dim3(threads), 0, stream, a);
    }
    constexpr int VEC = 16 / sizeof(R);
    const int nv = C / VEC;
    const int threads = nv >= 256 ? 256 : (nv >= 128 ? 128 : (nv >= 64 ? 64 : 32));
    const dim3 grid(a.max_count, (nv + threads - 1) / threads);
    switch (a.d_conv) {
#define SCONV_DC(n) \
    case n: return launch_pdl(extract_paged_vec<R, n>, grid, dim3(threads), 0, stream, a);
        SCONV_DC(1) SCONV_DC(2) SCONV_DC(3) SCONV_DC(4)
        SCONV_DC(5) SCONV_DC(6) SCONV_DC(7) SCONV_DC(8)
#undef SCONV_DC
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_scatter_ssm(const SsmArgs &a, int elem_bytes, bool vec, cudaStream_t stream) {
    if (vec) {
        const int64_t chunks = a.state_flat * elem_bytes / 16;
        const int threads = 256;
        const int64_t per_block = static_cast<int64_t>(threads) * kUnroll;
        const dim3 grid(static_cast<unsigned>((chunks + per_block - 1) / per_block), a.max_count);
        return launch_pdl(scatter_ssm_vec, grid, dim3(threads), 0, stream, a, chunks,
                          a.states_rs * elem_bytes / 16, a.out_rs * elem_bytes / 16);
    }
    const dim3 grid(static_cast<unsigned>((a.state_flat + 255) / 256), a.max_count);
    if (elem_bytes == 2) return launch_pdl(scatter_ssm_elem<uint16_t>, grid, dim3(256), 0, stream, a);
    return launch_pdl(scatter_ssm_elem<uint32_t>, grid, dim3(256), 0, stream, a);
}

cudaError_t launch_extract_paged(const PagedExtractArgs &a, bool bf16_data, bool vec,
                                 cudaStream_t stream) {
    return bf16_data ? launch_paged_t<uint16_t>(a, vec, stream)
                     : launch_paged_t<uint32_t>(a, vec, stream);
}

}  // namespace sconv
