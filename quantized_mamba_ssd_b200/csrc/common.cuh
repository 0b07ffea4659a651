// Device helpers shared by the SSD kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/ssd_i8.h"

namespace ssd {

constexpr int kWarp = 32;

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Output store in the requested dtype.  I8 applies q = clamp(rne(y * inv_scale), -127, 127)
// with inv_scale = 1 / y_scale computed once in fp32 on the host and the product rounded once
// (as in the chunk scan's epilogue).
__device__ __forceinline__ void store_out(void* y, size_t idx, float v, int dtype, float inv_scale) {
    if (dtype == SSD_OUT_F32) {
        static_cast<float*>(y)[idx] = v;
    } else if (dtype == SSD_OUT_F16) {
        static_cast<__half*>(y)[idx] = __float2half_rn(v);
    } else {
        // an FMA with 1.5 * 2^23 rounds the exact product to an integer, half to even
        // (|v * inv_scale| >= 2^22 lands outside +-127 either way and is clamped)
        constexpr float kRoundI = 12582912.f;
        float r = __fmaf_rn(v, inv_scale, kRoundI) - kRoundI;
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
