// Single-token SSD state update for decode (the "SSD update" the Quamba2 rebuttal measures at
// generation time, Tables R7/R8), one step of h_t = exp(dt A) h_{t-1} + dt x_t B_t^T,
// y_t = h_t C_t + D x_t, on an fp32 state held in HBM and updated in place.
//
// Pure streaming: the state is read once and written once with 16-byte accesses, and the
// output reduction over dstate runs in warp shuffles.  One CTA per (batch, head).
#include "common.cuh"
#include "ssd_kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;  // rows in flight per lane

template <int N, bool HAD>
__global__ void __launch_bounds__(kThreads)
state_update_kernel(float* __restrict__ state, const int8_t* __restrict__ x,
                    const int8_t* __restrict__ Bq, const int8_t* __restrict__ Cq,
                    const float* __restrict__ dt, const float* __restrict__ A,
                    const float* __restrict__ D, const float* __restrict__ x_scale,
                    const float* __restrict__ B_scale, const float* __restrict__ C_scale,
                    int H, int P, int G, int per_n, void* __restrict__ y, int y_dtype,
                    float inv_y_scale) {
    __shared__ float ys[HAD ? 64 : 1];  // y of this (batch, head) to be transformed (P = 64)
    constexpr int VEC = N / 4;                          // float4 per state row
    constexpr int LPR = VEC < kWarp ? VEC : kWarp;      // lanes per row
    constexpr int VPL = VEC / LPR;                      // float4 per lane per row
    constexpr int RPW = kWarp / LPR;                    // rows per warp pass
    const int h = blockIdx.x, b = blockIdx.y;
    const int g = h / (H / G);
    const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x / kWarp;
    const int sub = lane % LPR, rsub = lane / LPR;

    const float dtv = dt[(size_t)b * H + h];
    const float decay = __expf(dtv * A[h]);
    const float sx = x_scale[h], Dh = D[h];
    // B and C scales: per group, or per group and dstate channel (SSDi8 Table 10, per-P(N))
    const float* sBv = B_scale + (per_n ? (size_t)g * N : g);
    const float* sCv = C_scale + (per_n ? (size_t)g * N : g);
    const int sn = per_n ? 1 : 0;
    float bv[VPL][4], cv[VPL][4];
    const int8_t* brow = Bq + ((size_t)b * G + g) * N;
    const int8_t* crow = Cq + ((size_t)b * G + g) * N;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        const int n0 = (sub + k * LPR) * 4;
        const char4 b4 = *reinterpret_cast<const char4*>(brow + n0);
        const char4 c4 = *reinterpret_cast<const char4*>(crow + n0);
        const int i0 = sn * n0;
        bv[k][0] = sBv[i0] * b4.x; bv[k][1] = sBv[i0 + sn] * b4.y;
        bv[k][2] = sBv[i0 + 2 * sn] * b4.z; bv[k][3] = sBv[i0 + 3 * sn] * b4.w;
        cv[k][0] = sCv[i0] * c4.x; cv[k][1] = sCv[i0 + sn] * c4.y;
        cv[k][2] = sCv[i0 + 2 * sn] * c4.z; cv[k][3] = sCv[i0 + 3 * sn] * c4.w;
    }
    float4* st = reinterpret_cast<float4*>(state + ((size_t)b * H + h) * P * N);
    const int8_t* xrow = x + ((size_t)b * H + h) * P;
    const size_t ybase = ((size_t)b * H + h) * P;
    const int rows_per_pass = (kThreads / kWarp) * RPW;

    // the loop bound is warp-uniform so that every lane reaches the shuffles below
    for (int base = warp * RPW; base < P; base += rows_per_pass * kUnroll) {
        const int p0 = base + rsub;
        float4 hv[kUnroll][VPL];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int p = p0 + u * rows_per_pass;
#pragma unroll
            for (int k = 0; k < VPL; ++k)
                hv[u][k] = p < P ? st[(size_t)p * VEC + sub + k * LPR] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int p = p0 + u * rows_per_pass;
            const float xv = p < P ? sx * static_cast<float>(xrow[p]) : 0.f;
            const float dx = dtv * xv;
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < VPL; ++k) {
                float4 v = hv[u][k];
                v.x = fmaf(decay, v.x, dx * bv[k][0]);
                v.y = fmaf(decay, v.y, dx * bv[k][1]);
                v.z = fmaf(decay, v.z, dx * bv[k][2]);
                v.w = fmaf(decay, v.w, dx * bv[k][3]);
                acc = fmaf(cv[k][0], v.x, acc);
                acc = fmaf(cv[k][1], v.y, acc);
                acc = fmaf(cv[k][2], v.z, acc);
                acc = fmaf(cv[k][3], v.w, acc);
                if (p < P) st[(size_t)p * VEC + sub + k * LPR] = v;
            }
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (sub == 0 && p < P) {
                if constexpr (HAD) ys[p] = acc + Dh * xv;
                else store_out(y, ybase + p, acc + Dh * xv, y_dtype, inv_y_scale);
            }
        }
    }
    if constexpr (HAD) {
        __syncthreads();
        if (warp == 0) hadamard64_store(ys, y, ybase, y_dtype, inv_y_scale);
    }
}

template <int N>
cudaError_t launch_n(const StateUpdateArgs& a, cudaStream_t st) {
    dim3 grid(a.nheads, a.batch);
    auto kernel = a.hadamard ? state_update_kernel<N, true> : state_update_kernel<N, false>;
    kernel<<<grid, kThreads, 0, st>>>(a.state, a.x, a.B, a.C, a.dt, a.A, a.D, a.x_scale, a.B_scale,
                                      a.C_scale, a.nheads, a.headdim, a.ngroups, a.per_n, a.y,
                                      a.y_dtype, a.inv_y_scale);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_state_update(const StateUpdateArgs& a, cudaStream_t st) {
    switch (a.dstate) {
        case 16: return launch_n<16>(a, st);
        case 32: return launch_n<32>(a, st);
        case 64: return launch_n<64>(a, st);
        case 128: return launch_n<128>(a, st);
        case 256: return launch_n<256>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ssd
