// extract.cu -- conditional, transposed gather of length-d_conv conv windows
// for prefix caching ("core.ssm.ops.intermediate_extraction",
// _scatter_intermediate_conv_kernel / scatter_intermediate_conv), sm_100a.
//
// Grid: (max_count slots, channel blocks); sized at capture time from
// max_count and conv_dim only.  Each block reads the runtime real_count from
// device memory and returns at once when its slot is at or beyond it, so
// padded slots move no data.  A thread gathers the d_conv rows of one
// 16-byte channel pack and writes them transposed: out[slot][c][k] is
// contiguous in k, so the VEC channels x d_conv taps of a thread form one
// contiguous run of d_conv 16-byte stores.
#include "common.cuh"

namespace sconv {
namespace {

// Raw element type of the copy: the gather never interprets values.
template <typename E>
struct Raw;
template <>
struct Raw<float> {
    using T = uint32_t;
};
template <>
struct Raw<bf16> {
    using T = uint16_t;
};

__device__ __forceinline__ int clamped_count(const ExtractArgs &a) {
    if (threadIdx.x == 0) {  // while the preceding kernel drains
        prefetch_l2(a.real_count);
        prefetch_l2(a.abs_pos + blockIdx.x);
    }
    pdl_wait();
    pdl_trigger();
    int rc = __ldg(a.real_count);
    if (rc < 0) rc = 0;
    if (rc > a.max_count) rc = a.max_count;
    return rc;
}

// Before the PDL wait the thread reads real_count and its slot's end
// position *speculatively* (L2-only loads; the preceding kernel may still be
// writing them), range-checks them and only prefetches its window's rows
// into L2.  After the wait real_count and the end position are loaded
// together, so the gather waits for one L2 round trip before its rows, not
// two; a stale speculative value costs a useless prefetch, never a wrong
// result.
template <typename E, int DC>
__global__ void __launch_bounds__(256) extract_windows_vec(const __grid_constant__ ExtractArgs a) {
    using R = typename Raw<E>::T;
    constexpr int VEC = Elem<E>::kVec;
    const int slot = blockIdx.x;
    const int pack = blockIdx.y * blockDim.x + threadIdx.x;
    const bool in_range = pack < a.conv_dim / VEC;
    const int c = pack * VEC;
    const R *src = static_cast<const R *>(a.src);
    if (in_range && slot < __ldcg(a.real_count)) {
        const int64_t end = __ldcg(a.abs_pos + slot);
#pragma unroll
        for (int k = 0; k < DC; ++k) {
            const int64_t p = end - DC + k;
            if (p >= 0 && p < a.seq_len) prefetch_l2(src + p * a.src_ss + c);
        }
    }
    pdl_wait();
    pdl_trigger();
    int rc = __ldg(a.real_count);
    const int64_t end = __ldg(a.abs_pos + slot);  // slot < max_count: always in bounds
    if (rc > a.max_count) rc = a.max_count;
    if (slot >= rc || !in_range) return;

    union U {
        uint4 u;
        R e[VEC];
    };
    U rows[DC];
#pragma unroll
    for (int k = 0; k < DC; ++k) {
        const int64_t p = end - DC + k;
        if (p >= 0 && p < a.seq_len)
            rows[k].u = __ldg(reinterpret_cast<const uint4 *>(src + p * a.src_ss + c));
        else
            rows[k].u = make_uint4(0u, 0u, 0u, 0u);
    }
    // Transpose VEC x DC -> DC x VEC in registers: element (channel v, tap k)
    // goes to position v*DC + k of the thread's output run.
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

// Any layout: one thread per channel, element-wise copies.
template <typename E>
__global__ void __launch_bounds__(256) extract_windows_scalar(const __grid_constant__ ExtractArgs a,
                                                              int64_t src_sc) {
    using R = typename Raw<E>::T;
    const int slot = blockIdx.x;
    if (slot >= clamped_count(a)) return;
    const int c = blockIdx.y * blockDim.x + threadIdx.x;
    if (c >= a.conv_dim) return;
    const int64_t end = __ldg(a.abs_pos + slot);
    const R *src = static_cast<const R *>(a.src);
    R *dst = static_cast<R *>(a.out) + slot * a.out_ss + static_cast<int64_t>(c) * a.d_conv;
    for (int k = 0; k < a.d_conv; ++k) {
        const int64_t p = end - a.d_conv + k;
        dst[k] = (p >= 0 && p < a.seq_len) ? __ldg(src + p * a.src_ss + c * src_sc) : R(0);
    }
}

template <typename E>
cudaError_t launch_vec(const ExtractArgs &a, cudaStream_t stream) {
    constexpr int VEC = Elem<E>::kVec;
    const int nv = a.conv_dim / VEC;
    const int threads = nv >= 256 ? 256 : (nv >= 128 ? 128 : (nv >= 64 ? 64 : 32));
    dim3 grid(a.max_count, (nv + threads - 1) / threads);
    switch (a.d_conv) {
#define SCONV_DC(n) \
    case n: return launch_pdl(extract_windows_vec<E, n>, grid, dim3(threads), 0, stream, a);
        SCONV_DC(1) SCONV_DC(2) SCONV_DC(3) SCONV_DC(4)
        SCONV_DC(5) SCONV_DC(6) SCONV_DC(7) SCONV_DC(8)
#undef SCONV_DC
        default: return cudaErrorInvalidValue;
    }
}

template <typename E>
cudaError_t launch_scalar(const ExtractArgs &a, int64_t src_sc, cudaStream_t stream) {
    const int threads = a.conv_dim >= 256 ? 256 : 64;
    dim3 grid(a.max_count, (a.conv_dim + threads - 1) / threads);
    return launch_pdl(extract_windows_scalar<E>, grid, dim3(threads), 0, stream, a, src_sc);
}

}  // namespace

cudaError_t launch_extract(const ExtractArgs &a, bool bf16_data, bool vec, cudaStream_t stream) {
    if (bf16_data) return vec ? launch_vec<bf16>(a, stream) : launch_scalar<bf16>(a, 1, stream);
    return vec ? launch_vec<float>(a, stream) : launch_scalar<float>(a, 1, stream);
}

}  // namespace sconv
