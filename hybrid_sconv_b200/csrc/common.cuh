// common.cuh -- shared device helpers of the sconv library (sm_100a).
//
// Data moves in "packs": VEC consecutive channel elements of one row that
// travel as a single 16-byte transaction (8 bf16 or 4 fp32), or as one
// element when a layout is not 16-byte aligned.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sconv {

using bf16 = __nv_bfloat16;

template <typename E>
struct Elem;
template <>
struct Elem<float> {
    static constexpr int kVec = 4;  // elements per 16-byte pack
};
template <>
struct Elem<bf16> {
    static constexpr int kVec = 8;
};

// VEC elements of type E held in registers as raw bits.
template <typename E, int VEC>
struct Pack;

// 16-byte pack: four 32-bit words.
template <typename E>
struct Pack16 {
    uint4 u;
    __device__ __forceinline__ void load_nc(const E *p) {
        u = __ldg(reinterpret_cast<const uint4 *>(p));
    }
    __device__ __forceinline__ void store(E *p) const {
        *reinterpret_cast<uint4 *>(p) = u;
    }
    __device__ __forceinline__ void zero() { u = make_uint4(0u, 0u, 0u, 0u); }
};

template <>
struct Pack<bf16, 8> : Pack16<bf16> {
    // bf16 is the upper half of an fp32, so the widening is exact.
    __device__ __forceinline__ void to_float(float (&f)[8]) const {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ void from_float(const float (&f)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t *>(&h);
        }
        u = make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <>
struct Pack<float, 4> : Pack16<float> {
    __device__ __forceinline__ void to_float(float (&f)[4]) const {
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
    }
    __device__ __forceinline__ void from_float(const float (&f)[4]) {
        u = make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                       __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};

// One-element packs for layouts that are not 16-byte aligned.
template <>
struct Pack<float, 1> {
    float v;
    __device__ __forceinline__ void load_nc(const float *p) { v = __ldg(p); }
    __device__ __forceinline__ void store(float *p) const { *p = v; }
    __device__ __forceinline__ void zero() { v = 0.f; }
    __device__ __forceinline__ void to_float(float (&f)[1]) const { f[0] = v; }
    __device__ __forceinline__ void from_float(const float (&f)[1]) { v = f[0]; }
};

template <>
struct Pack<bf16, 1> {
    unsigned short v;
    __device__ __forceinline__ void load_nc(const bf16 *p) {
        v = __ldg(reinterpret_cast<const unsigned short *>(p));
    }
    __device__ __forceinline__ void store(bf16 *p) const {
        *reinterpret_cast<unsigned short *>(p) = v;
    }
    __device__ __forceinline__ void zero() { v = 0; }
    __device__ __forceinline__ void to_float(float (&f)[1]) const {
        f[0] = __uint_as_float(static_cast<uint32_t>(v) << 16);
    }
    __device__ __forceinline__ void from_float(const float (&f)[1]) {
        bf16 h = __float2bfloat16_rn(f[0]);
        v = *reinterpret_cast<unsigned short *>(&h);
    }
};

__device__ __forceinline__ float load_weight(const float *p) { return __ldg(p); }
__device__ __forceinline__ float load_weight(const bf16 *p) {
    return __uint_as_float(
        static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short *>(p))) << 16);
}

// Arguments of one fused launch, validated on the host.  Strides in elements.
struct FusedArgs {
    const void *x;
    int64_t x_rs;
    int T, C;
    const void *w;
    int64_t w_sc, w_sk;
    int W;
    void *cache;
    int64_t cs0, cs1, cs2;  // block, head, offset strides (D stride is 1)
    int64_t num_blocks;
    int H, N, D;
    const int64_t *positions;
    const int32_t *seq_idx;  // unused when every token is its own request
    const int64_t *slot;
    const int32_t *qstart;   // unused when every token is its own request
    const int32_t *bt;
    int64_t bt_rs;
    int num_reqs, max_blocks;
    int off_s, ws;
    int silu, resid;
    void *out;
    int64_t out_rs;
    int32_t *err;
};

struct ExtractArgs {
    const void *src;
    int64_t seq_len;
    int conv_dim;
    int64_t src_ss;
    const int32_t *abs_pos;
    const int32_t *real_count;
    int max_count;
    void *out;
    int64_t out_ss;
    int d_conv;
};

// Host-side launchers (return the cudaError_t of the launch).
cudaError_t launch_fused(const FusedArgs &a, bool bf16_data, bool vec, bool one_token_per_request,
                         cudaStream_t stream);
cudaError_t launch_extract(const ExtractArgs &a, bool bf16_data, bool vec, cudaStream_t stream);
cudaError_t launch_seq_metadata(const int32_t *qsl, int num_reqs, int num_actual, int num_padded,
                                int32_t *seq_idx, int32_t *query_start, cudaStream_t stream);

}  // namespace sconv
