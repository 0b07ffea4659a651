// Device helpers shared by the SSD kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/ssd_i8.h"

namespace ssd {

constexpr int kWarp = 32;

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// int8 x int8 dot product of 4 lanes accumulated in int32 (exact).
__device__ __forceinline__ int dot4_i8(int a, int b, int acc) { return __dp4a(a, b, acc); }

// Inclusive prefix sum over one warp (shuffle-up scan).
__device__ __forceinline__ float warp_inclusive_scan(float v) {
    const int lane = threadIdx.x & (kWarp - 1);
#pragma unroll
    for (int o = 1; o < kWarp; o <<= 1) {
        float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = kWarp / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Inclusive block-wide prefix sum of one value per thread; `scratch` holds >= 32 floats.
// Every thread of the block must call it.
__device__ __forceinline__ float block_inclusive_scan(float v, float* scratch) {
    const int lane = threadIdx.x & (kWarp - 1);
    const int warp = threadIdx.x / kWarp;
    const int nwarps = blockDim.x / kWarp;
    v = warp_inclusive_scan(v);
    if (lane == kWarp - 1) scratch[warp] = v;
    __syncthreads();
    if (warp == 0) {
        float w = lane < nwarps ? scratch[lane] : 0.f;
        w = warp_inclusive_scan(w);
        if (lane < nwarps) scratch[lane] = w;
    }
    __syncthreads();
    if (warp > 0) v += scratch[warp - 1];
    __syncthreads();
    return v;
}

// Output store in the requested dtype.  I8 applies q = clamp(rne(y * inv_scale), -127, 127)
// with inv_scale = 1 / y_scale computed once in fp32 on the host.
__device__ __forceinline__ void store_out(void* y, size_t idx, float v, int dtype, float inv_scale) {
    if (dtype == SSD_OUT_F32) {
        static_cast<float*>(y)[idx] = v;
    } else if (dtype == SSD_OUT_F16) {
        static_cast<__half*>(y)[idx] = __float2half_rn(v);
    } else {
        float r = rintf(v * inv_scale);
        r = fminf(fmaxf(r, -127.f), 127.f);
        static_cast<int8_t*>(y)[idx] = static_cast<int8_t>(static_cast<int>(r));
    }
}

// y' = H y / 8 of the 64 values ys[0..63] (H the Sylvester-ordered 64 x 64 Hadamard matrix,
// H = [[H32, H32], [H32, -H32]]), stored at y[ybase + q] in the output dtype.  Called by one
// whole warp: lane l holds y'[l] = H32 (y_lo + y_hi) and y'[l + 32] = H32 (y_lo - y_hi), the
// 32-point transforms as five butterfly stages across the lanes.
__device__ __forceinline__ void hadamard64_store(const float* ys, void* y, size_t ybase, int dtype,
                                                 float inv_scale) {
    const int lane = threadIdx.x & (kWarp - 1);
    const float a = ys[lane], b = ys[lane + 32];
    float s = a + b, d = a - b;
#pragma unroll
    for (int hs = 16; hs >= 1; hs >>= 1) {
        const float ps = __shfl_xor_sync(0xffffffffu, s, hs);
        const float pd = __shfl_xor_sync(0xffffffffu, d, hs);
        const bool upper = (lane & hs) != 0;  // element i + hs of the butterfly (i, i + hs)
        s = upper ? ps - s : s + ps;
        d = upper ? pd - d : d + pd;
    }
    store_out(y, ybase + lane, 0.125f * s, dtype, inv_scale);
    store_out(y, ybase + lane + 32, 0.125f * d, dtype, inv_scale);
}

}  // namespace ssd
