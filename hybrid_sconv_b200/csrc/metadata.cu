// metadata.cu -- per-token request index and request start in one launch
// ("vllm.models.inkling.nvidia.ops.sconv", sconv_seq_metadata), sm_100a.
//
// One thread per token row.  The request is the last r < num_reqs with
// query_start_loc[r] <= t, found by binary search; when the offsets table
// is small each block first stages it in shared memory so the search's
// dependent loads hit shared memory instead of L2.  A second entry point
// runs the same lookup ahead of its wait on the stream.  A third kernel
// also resolves every token's pre-forward taps into a table.
#include "common.cuh"
#include "sconv.h"
#include "taps_resolve.cuh"

namespace sconv {
namespace {

constexpr int kThreads = 256;
constexpr int kSmemReqs = 4096;  // stage query_start_loc when num_reqs <= this

// AHEAD = false waits for the kernels before it on the stream, then works.
// AHEAD = true works first and waits at its end: its completion, which the
// next kernel waits for, still follows theirs, while the lookup overlaps
// them.  It is valid only when none of the kernels that may still be running
// writes query_start_loc or touches the two outputs (one metadata buffer set
// per step in flight).
template <bool AHEAD>
__global__ void __launch_bounds__(kThreads)
seq_metadata_kernel(const int32_t *__restrict__ qsl, int num_reqs, int num_actual,
                    int num_padded, int32_t *__restrict__ seq_idx,
                    int32_t *__restrict__ query_start, int staged) {
    extern __shared__ int32_t s_qsl[];
    // Let the next kernel (typically the fused step that reads these
    // buffers) launch at once: its own wait still orders it after this
    // kernel, and it gets this kernel's whole wait to prefetch.  Then pull
    // the offsets table into L2 while the preceding kernel drains.
    pdl_trigger();
    if (!AHEAD) {
        for (int i = threadIdx.x * 32; i < num_reqs; i += blockDim.x * 32) prefetch_l2(qsl + i);
        pdl_wait();
    }
    if (staged) {
        for (int i = threadIdx.x; i < num_reqs; i += blockDim.x) s_qsl[i] = __ldg(qsl + i);
        __syncthreads();
    }
    const int32_t *q = staged ? s_qsl : qsl;
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t < num_padded) {
        if (t >= num_actual) {
            seq_idx[t] = 0;
            query_start[t] = 0;
        } else {
            // Invariant: the answer lies in [lo, hi]; q[lo] <= t is assumed for lo = 0.
            int lo = 0, hi = num_reqs - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (q[mid] <= t) lo = mid;
                else hi = mid - 1;
            }
            seq_idx[t] = lo;
            query_start[t] = q[lo];
        }
    }
    if (AHEAD) pdl_wait();  // every thread: the grid completes after its predecessor
}

// The standalone tap resolution (taps_resolve.cuh), one thread per token.
template <bool AHEAD, bool DECODE, int MAXW>
__global__ void __launch_bounds__(kThreads) seq_metadata_taps_kernel(const TapResolveArgs a) {
    extern __shared__ int32_t s_qsl[];
    pdl_trigger();  // as in seq_metadata_kernel
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (!AHEAD) {
        if (!DECODE)
            for (int i = threadIdx.x * 32; i < a.num_reqs; i += blockDim.x * 32)
                prefetch_l2(a.qsl + i);
        if (t < a.num_actual && (threadIdx.x & 15) == 0) {
            prefetch_l2(a.positions + t);
            prefetch_l2(a.slot + t);
        }
        pdl_wait();
    }
    resolve_block<DECODE, MAXW>(a, t, threadIdx.x, blockDim.x, s_qsl);
    if (AHEAD) pdl_wait();  // every thread: the grid completes after its predecessor
}

template <bool AHEAD, bool DECODE>
cudaError_t launch_taps_w(const TapResolveArgs &a, size_t smem, cudaStream_t stream) {
    const int blocks = (a.num_padded + kThreads - 1) / kThreads;
    if (a.W <= 4)
        return launch_pdl(seq_metadata_taps_kernel<AHEAD, DECODE, 4>, dim3(blocks),
                          dim3(kThreads), smem, stream, a);
    return launch_pdl(seq_metadata_taps_kernel<AHEAD, DECODE, 8>, dim3(blocks), dim3(kThreads),
                      smem, stream, a);
}

}  // namespace

cudaError_t launch_seq_metadata_taps(TapResolveArgs &a, bool ahead, cudaStream_t stream) {
    size_t smem = 0;
    resolve_staging(a, smem);
    const bool decode = a.qsl == nullptr;
    if (ahead)
        return decode ? launch_taps_w<true, true>(a, smem, stream)
                      : launch_taps_w<true, false>(a, smem, stream);
    return decode ? launch_taps_w<false, true>(a, smem, stream)
                  : launch_taps_w<false, false>(a, smem, stream);
}

cudaError_t launch_seq_metadata(const int32_t *qsl, int num_reqs, int num_actual, int num_padded,
                                int32_t *seq_idx, int32_t *query_start, bool ahead,
                                cudaStream_t stream) {
    // With no actual tokens the search never runs; one entry keeps the
    // staging loop and the search bounds well defined.
    const int nr = num_reqs > 0 ? num_reqs : 1;
    const int staged = nr <= kSmemReqs ? 1 : 0;
    const size_t smem = staged ? static_cast<size_t>(nr) * sizeof(int32_t) : 0;
    const int blocks = (num_padded + kThreads - 1) / kThreads;
    if (ahead)
        return launch_pdl(seq_metadata_kernel<true>, dim3(blocks), dim3(kThreads), smem, stream,
                          qsl, nr, num_actual, num_padded, seq_idx, query_start, staged);
    return launch_pdl(seq_metadata_kernel<false>, dim3(blocks), dim3(kThreads), smem, stream, qsl,
                      nr, num_actual, num_padded, seq_idx, query_start, staged);
}

}  // namespace sconv
