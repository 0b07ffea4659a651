// Decode with an int8 cached SSM state (the quantized cached state of the Quamba2 rebuttal's
// generation-time discussion, Tables R7/R8): the state of one (batch, head) is int8 codes
// [headdim][dstate] with one fp32 scale, h = scale * code.  One step dequantises, applies
// h_t = exp(dt A) h_{t-1} + dt x_t B_t^T and y_t = h_t C_t + D x_t in fp32, then requantises
// h_t with the symmetric per-(batch, head) rule scale = max|h_t| / 127,
// code = clamp(round_half_even(h_t / scale), -127, 127).
//
// One CTA per (batch, head); every thread keeps its 16-byte chunks of the state in registers
// between the update and the requantisation (the scale needs the maximum over the whole state
// first).  The state moves once in each direction at one byte per element.
#include <type_traits>

#include "common.cuh"
#include "ssd_kernels.h"

namespace ssd {

namespace {

// CTA size TPB and 16-byte state chunks per thread CH are chosen per shape (launch_*_shape):
// small CTAs with a few chunks each keep many CTAs, and their loads, in flight per SM
constexpr int kMaxThreads = 256;
constexpr int kMaxChunksPerThread = 4;  // headdim * dstate <= 16384

// 16 int8 codes (one 16-byte chunk) -> 16 floats, exactly and on the full-rate pipes: the
// byte (sign bit flipped) becomes the low mantissa byte of 2^23, and 2^23 + 128 comes off again
__device__ __forceinline__ void unpack16(const uint4 w, float (&v)[16]) {
    const uint32_t ww[4] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u, w.z ^ 0x80808080u,
                            w.w ^ 0x80808080u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[4 * i + 0] = __uint_as_float(__byte_perm(ww[i], 0x4B000000u, 0x7540)) - 8388736.f;
        v[4 * i + 1] = __uint_as_float(__byte_perm(ww[i], 0x4B000000u, 0x7541)) - 8388736.f;
        v[4 * i + 2] = __uint_as_float(__byte_perm(ww[i], 0x4B000000u, 0x7542)) - 8388736.f;
        v[4 * i + 3] = __uint_as_float(__byte_perm(ww[i], 0x4B000000u, 0x7543)) - 8388736.f;
    }
}

// q = rne(fp32(v * inv)) of 16 values -> one 16-byte chunk, for inv = 127 / max|v| taken over the
// same fp32 values: then |v * inv| <= 127 (1 + 2^-22) < 127.5, so no clamp is needed.  Adding
// 1.5 * 2^23 rounds to an integer (half to even) in the low mantissa bits, whose low byte is then
// the code.
__device__ __forceinline__ uint4 pack16(const float (&v)[16], float inv) {
    constexpr float kRound = 12582912.f;
    uint32_t ww[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t c[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            c[j] = __float_as_uint(__fadd_rn(__fmul_rn(v[4 * i + j], inv), kRound));  // no contraction
        ww[i] = __byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x0040), 0x5410);
    }
    return make_uint4(ww[0], ww[1], ww[2], ww[3]);
}

// max over the CTA (every thread calls it; `scratch` holds TPB / 32 floats)
template <int TPB>
__device__ __forceinline__ float block_max(float v, float* scratch) {
#pragma unroll
    for (int o = kWarp / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int lane = threadIdx.x & (kWarp - 1), warp = threadIdx.x / kWarp;
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    float m = 0.f;
#pragma unroll
    for (int w = 0; w < TPB / kWarp; ++w) m = fmaxf(m, scratch[w]);
    return m;
}

template <int N, int TPB, int CH>
__global__ void __launch_bounds__(TPB)
state_update_q8_kernel(int8_t* __restrict__ state_q, float* __restrict__ state_scale,
                       const int8_t* __restrict__ x, const int8_t* __restrict__ Bq,
                       const int8_t* __restrict__ Cq, const float* __restrict__ dt,
                       const float* __restrict__ A, const float* __restrict__ D,
                       const float* __restrict__ x_scale, const float* __restrict__ B_scale,
                       const float* __restrict__ C_scale, int H, int P, int G,
                       void* __restrict__ y, int y_dtype, float inv_y_scale) {
    constexpr int CPR = N / 16;  // 16-byte chunks per state row (lanes per row, <= 16)
    __shared__ float scratch[TPB / kWarp];
    __shared__ __align__(16) float sbv[N], scv[N];  // s_B B_n and s_C C_n of this (batch, group)
    const int h = blockIdx.x, b = blockIdx.y;
    const int g = h / (H / G);
    const int tid = threadIdx.x, lane = tid & (kWarp - 1);
    const size_t bh = (size_t)b * H + h;
    const int nchunks = P * CPR;

    const int8_t* brow = Bq + ((size_t)b * G + g) * N;
    const int8_t* crow = Cq + ((size_t)b * G + g) * N;
    const int8_t* xrow = x + bh * P;
    uint4* st = reinterpret_cast<uint4*>(state_q + bh * P * N);
    // every global load of the step is issued here, before anything waits on one: the codes
    // (they stay in registers, a quarter of the floats; the update is recomputed for the
    // requantisation, so registers, not ALU work, bound the CTAs with loads in flight), the
    // token's x of this thread's rows, and the scalars
    uint4 qv[CH];
    float xq[CH];
#pragma unroll
    for (int k = 0; k < CH; ++k) {
        const int u = tid + k * TPB;
        const bool in = k * TPB < nchunks && u < nchunks;
        qv[k] = in ? st[u] : make_uint4(0u, 0u, 0u, 0u);
        xq[k] = in ? static_cast<float>(xrow[u / CPR]) : 0.f;
    }
    const float dtv = dt[bh];
    const float decay = __expf(dtv * A[h]);
    const float s_old = state_scale[bh];
    const float sx = x_scale[h], sB = B_scale[g], sC = C_scale[g], Dh = D[h];
    if (tid < 2 * CPR) {
        const int cc = tid % CPR;
        float v[16];
        unpack16(*reinterpret_cast<const uint4*>((tid < CPR ? brow : crow) + 16 * cc), v);
        float* dst = (tid < CPR ? sbv : scv) + 16 * cc;
        const float sc = tid < CPR ? sB : sC;
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[i] = sc * v[i];
    }
    __syncthreads();

    const float ds = decay * s_old;  // decayed dequantisation factor
    float amax = 0.f;
    // the loop bound is warp-uniform (multiples of the CTA size) so that every lane reaches
    // the shuffles
#pragma unroll
    for (int k = 0; k < CH; ++k) {
        if (k * TPB >= nchunks) break;
        const int u = tid + k * TPB;
        const bool in = u < nchunks;
        const int p = in ? u / CPR : 0, cc = u % CPR;
        const float4* bq4 = reinterpret_cast<const float4*>(sbv + 16 * cc);
        const float4* cq4 = reinterpret_cast<const float4*>(scv + 16 * cc);
        float hv[16];
        unpack16(qv[k], hv);
        const float xv = sx * xq[k];
        const float dx = dtv * xv;
        float acc = 0.f;
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
            const float4 b4 = bq4[i4], c4 = cq4[i4];
            const float bb[4] = {b4.x, b4.y, b4.z, b4.w}, cc4[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float v = fmaf(ds, hv[4 * i4 + j], dx * bb[j]);
                acc = fmaf(cc4[j], v, acc);
                amax = fmaxf(amax, fabsf(v));
            }
        }
#pragma unroll
        for (int o = CPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (in && (lane % CPR) == 0) store_out(y, bh * P + p, acc + Dh * xv, y_dtype, inv_y_scale);
    }
    amax = block_max<TPB>(amax, scratch);
    const float inv = amax > 0.f ? 127.f / amax : 0.f;
#pragma unroll
    for (int k = 0; k < CH; ++k) {
        if (k * TPB >= nchunks) break;
        const int u = tid + k * TPB;
        if (u >= nchunks) continue;
        const int cc = u % CPR;
        const float4* bq4 = reinterpret_cast<const float4*>(sbv + 16 * cc);
        const float dx = dtv * (sx * xq[k]);
        float hv[16];
        unpack16(qv[k], hv);
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
            const float4 b4 = bq4[i4];
            hv[4 * i4 + 0] = fmaf(ds, hv[4 * i4 + 0], dx * b4.x);
            hv[4 * i4 + 1] = fmaf(ds, hv[4 * i4 + 1], dx * b4.y);
            hv[4 * i4 + 2] = fmaf(ds, hv[4 * i4 + 2], dx * b4.z);
            hv[4 * i4 + 3] = fmaf(ds, hv[4 * i4 + 3], dx * b4.w);
        }
        st[u] = pack16(hv, inv);
    }
    if (tid == 0) state_scale[bh] = amax / 127.f;
}

// fp32 state -> int8 codes + per-(batch, head) scale (the same rule as the update's requant)
template <int N, int TPB, int CH>
__global__ void __launch_bounds__(TPB)
state_quantize_kernel(const float* __restrict__ state, int8_t* __restrict__ state_q,
                      float* __restrict__ state_scale, int P) {
    constexpr int CPR = N / 16;
    __shared__ float scratch[TPB / kWarp];
    const size_t bh = blockIdx.x;
    const int tid = threadIdx.x;
    const int nchunks = P * CPR;
    const float4* src = reinterpret_cast<const float4*>(state + bh * P * N);
    uint4* dst = reinterpret_cast<uint4*>(state_q + bh * P * N);
    float hv[CH][16];
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < CH; ++k) {
        if (k * TPB >= nchunks) break;
        const int u = tid + k * TPB;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 f = u < nchunks ? src[4 * u + i] : make_float4(0.f, 0.f, 0.f, 0.f);
            hv[k][4 * i + 0] = f.x;
            hv[k][4 * i + 1] = f.y;
            hv[k][4 * i + 2] = f.z;
            hv[k][4 * i + 3] = f.w;
            amax = fmaxf(fmaxf(amax, fabsf(f.x)), fmaxf(fabsf(f.y), fmaxf(fabsf(f.z), fabsf(f.w))));
        }
    }
    amax = block_max<TPB>(amax, scratch);
    const float inv = amax > 0.f ? 127.f / amax : 0.f;
#pragma unroll
    for (int k = 0; k < CH; ++k) {
        if (k * TPB >= nchunks) break;
        const int u = tid + k * TPB;
        if (u < nchunks) dst[u] = pack16(hv[k], inv);
    }
    if (tid == 0) state_scale[bh] = amax / 127.f;
}

// (TPB, CH) for a state of `nchunks` 16-byte chunks: 128 threads while 4 chunks each suffice
template <typename F>
cudaError_t with_shape(int nchunks, F&& f) {
    if (nchunks <= 128) return f(std::integral_constant<int, 128>(), std::integral_constant<int, 1>());
    if (nchunks <= 256) return f(std::integral_constant<int, 128>(), std::integral_constant<int, 2>());
    if (nchunks <= 512) return f(std::integral_constant<int, 128>(), std::integral_constant<int, 4>());
    return f(std::integral_constant<int, 256>(), std::integral_constant<int, 4>());
}

template <int N>
cudaError_t launch_q8_n(const StateUpdateQ8Args& a, cudaStream_t st) {
    dim3 grid(a.nheads, a.batch);
    return with_shape(a.headdim * N / 16, [&](auto tpb, auto ch) {
        state_update_q8_kernel<N, decltype(tpb)::value, decltype(ch)::value>
            <<<grid, decltype(tpb)::value, 0, st>>>(
                a.state_q, a.state_scale, a.x, a.B, a.C, a.dt, a.A, a.D, a.x_scale, a.B_scale,
                a.C_scale, a.nheads, a.headdim, a.ngroups, a.y, a.y_dtype, a.inv_y_scale);
        return cudaGetLastError();
    });
}

template <int N>
cudaError_t launch_quantize_n(const float* state, int8_t* q, float* scale, int count, int P,
                              cudaStream_t st) {
    return with_shape(P * N / 16, [&](auto tpb, auto ch) {
        state_quantize_kernel<N, decltype(tpb)::value, decltype(ch)::value>
            <<<count, decltype(tpb)::value, 0, st>>>(state, q, scale, P);
        return cudaGetLastError();
    });
}

}  // namespace

bool state_q8_shape_ok(int headdim, int dstate) {
    return (dstate == 16 || dstate == 32 || dstate == 64 || dstate == 128 || dstate == 256) &&
           headdim >= 1 && headdim * dstate <= kMaxChunksPerThread * kMaxThreads * 16;
}

cudaError_t launch_state_update_q8(const StateUpdateQ8Args& a, cudaStream_t st) {
    switch (a.dstate) {
        case 16: return launch_q8_n<16>(a, st);
        case 32: return launch_q8_n<32>(a, st);
        case 64: return launch_q8_n<64>(a, st);
        case 128: return launch_q8_n<128>(a, st);
        case 256: return launch_q8_n<256>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_state_quantize(const float* state, int8_t* q, float* scale, int count,
                                  int headdim, int dstate, cudaStream_t st) {
    switch (dstate) {
        case 16: return launch_quantize_n<16>(state, q, scale, count, headdim, st);
        case 32: return launch_quantize_n<32>(state, q, scale, count, headdim, st);
        case 64: return launch_quantize_n<64>(state, q, scale, count, headdim, st);
        case 128: return launch_quantize_n<128>(state, q, scale, count, headdim, st);
        case 256: return launch_quantize_n<256>(state, q, scale, count, headdim, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ssd
