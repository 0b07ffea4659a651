// Decode with an int8 cached SSM state (the quantized cached state of the Quamba2 rebuttal's
// generation-time discussion, Tables R7/R8): the state of one (batch, head) is int8 codes
// [headdim][dstate] with one fp32 scale, h = scale * code.  One step dequantises, applies
// h_t = exp(dt A) h_{t-1} + dt x_t B_t^T and y_t = h_t C_t + D x_t in fp32, then requantises
// h_t with the symmetric per-(batch, head) rule scale = max|h_t| / 127,
// code = clamp(round_half_even(h_t / scale), -127, 127).
//
// Persistent CTAs walk the (batch, head) items.  Each thread stages its 16-byte chunks of the
// next item's codes (and a B or C chunk) with cp.async while the current item is computed, then
// runs two passes over the staged codes: the update with y and max|h_t|, and, once the CTA has
// the maximum, the same update again with the requantisation.  The state moves once in each
// direction at one byte per element.
#include <type_traits>

#include "common.cuh"
#include "ssd_kernels.h"

namespace ssd {

namespace {

// CTA size TPB and 16-byte state chunks per thread CH are chosen per shape (launch_*_shape):
// small CTAs with a few chunks each keep many CTAs, and their loads, in flight per SM
constexpr int kMaxThreads = 256;
constexpr int kMaxChunksPerThread = 4;  // headdim * dstate <= 16384

// packed fp32 pairs: one instruction for two lanes of work on sm_100
struct f2 {
    float x, y;
};

__device__ __forceinline__ f2 fmul2(f2 a, f2 b) {
    f2 r;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

__device__ __forceinline__ f2 fadd2(f2 a, f2 b) {
    f2 r;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return r;
}

// a * b + c, one rounding
__device__ __forceinline__ f2 ffma2(f2 a, f2 b, f2 c) {
    f2 r;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(r.x), "=f"(r.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return r;
}

// max(m, |a.x|, |a.y|): one three-input maximum
__device__ __forceinline__ float amax3(float m, f2 a) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(m), "f"(fabsf(a.x)), "f"(fabsf(a.y)));
    return r;
}

// 16 int8 codes (one 16-byte chunk) -> 8 pairs of floats, exactly: the byte (sign bit flipped)
// becomes the low mantissa byte of 2^23, and 2^23 + 128 comes off again (one packed subtract
// per pair)
__device__ __forceinline__ void unpack16(const uint4 w, f2 (&v)[8]) {
    const uint32_t ww[4] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u, w.z ^ 0x80808080u,
                            w.w ^ 0x80808080u};
    const f2 off = {-8388736.f, -8388736.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = fadd2(f2{__uint_as_float(__byte_perm(ww[i], 0x4B000000u, 0x7540)),
                            __uint_as_float(__byte_perm(ww[i], 0x4B000000u, 0x7541))}, off);
        v[2 * i + 1] = fadd2(f2{__uint_as_float(__byte_perm(ww[i], 0x4B000000u, 0x7542)),
                                __uint_as_float(__byte_perm(ww[i], 0x4B000000u, 0x7543))}, off);
    }
}

// q = rne(v * inv) of 16 values -> one 16-byte chunk, for inv = 127 / max|v| taken over the same
// fp32 values: then |v * inv| <= 127 (1 + 2^-22) < 127.5, so no clamp is needed.  Adding
// 1.5 * 2^23 rounds to an integer (half to even) in the low mantissa bits, whose low byte is then
// the code; the multiply and the add are one FMA (one rounding, of the exact product).
__device__ __forceinline__ uint4 pack16_fma(const f2 (&v)[8], float inv) {
    const f2 i2 = {inv, inv}, rnd = {12582912.f, 12582912.f};
    uint32_t ww[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const f2 a = ffma2(v[2 * i], i2, rnd), b = ffma2(v[2 * i + 1], i2, rnd);
        ww[i] = __byte_perm(__byte_perm(__float_as_uint(a.x), __float_as_uint(a.y), 0x0040),
                            __byte_perm(__float_as_uint(b.x), __float_as_uint(b.y), 0x0040), 0x5410);
    }
    return make_uint4(ww[0], ww[1], ww[2], ww[3]);
}

// the same rule for the fp32 quantiser, with the multiply and the add rounded separately (the
// documented rule: rne of the fp32 product)
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

// 16-byte asynchronous copy global -> shared (bypasses L1), and its group fences
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int K>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(K) : "memory"); }

// (batch, head, group) of an item, and r = head % (heads per group); stepping it by the grid
// stride needs no integer division (those cost tens of instructions each)
struct ItemPos {
    int b, h, g, r;
};

// Persistent CTAs, each walking the (batch, head) items blockIdx.x, + gridDim.x, ...  Every
// thread copies its own 16-byte state chunks (and the B or C chunk it stages) of the NEXT item
// into its private slots of a two-stage shared buffer while it computes the current one, so
// the loads stay in flight without holding registers.  The requantisation pass recomputes the
// update from the codes in shared memory: that costs a fifth more instructions than keeping it
// in registers, but the smaller register budget fits six CTAs per SM instead of four, and the
// step is bound by latency more than by issue.
template <int N, int TPB, int CH, bool HAD>
__global__ void __launch_bounds__(TPB, 768 / TPB)  // 24 warps per SM
state_update_q8_kernel(int8_t* __restrict__ state_q, float* __restrict__ state_scale,
                       const int8_t* __restrict__ x, const int8_t* __restrict__ Bq,
                       const int8_t* __restrict__ Cq, const float* __restrict__ dt,
                       const float* __restrict__ A, const float* __restrict__ D,
                       const float* __restrict__ x_scale, const float* __restrict__ B_scale,
                       const float* __restrict__ C_scale, int count, int H, int P, int G,
                       int per_n, void* __restrict__ y, int y_dtype, float inv_y_scale) {
    constexpr int CPR = N / 16;  // 16-byte chunks per state row (lanes per row, <= 16)
    __shared__ float scratch[TPB / kWarp];
    // s_B B_n and s_C C_n (double-buffered), float4 j of chunk cc at [j * CPR + cc]: the lanes
    // of a warp read consecutive 16-byte words (chunk cc of state row p pairs with B, C chunk cc)
    __shared__ __align__(16) float4 sbv[2][N / 4], scv[2][N / 4];
    // copies in flight: [stage][chunk k][thread] state chunks, [stage][thread < 2 CPR] B/C chunks
    __shared__ __align__(16) uint4 sq[2][CH][TPB];
    __shared__ __align__(16) uint4 sbc[2][2 * CPR];
    // y of the current item when it is Hadamard-transformed (P = 64); it is rewritten only
    // after the next item's staging barrier, which the transforming warp 0 reaches last
    __shared__ float ys[HAD ? 64 : 1];
    const int tid = threadIdx.x, lane = tid & (kWarp - 1);
    const int nchunks = P * CPR;
    int item = blockIdx.x;
    if (item >= count) return;
    // the item's position, and the stride's (the only divisions of the kernel)
    const int HG = H / G;
    const int Sb = gridDim.x / H, Sh = gridDim.x % H, Sg = Sh / HG, Sr = Sh % HG;
    ItemPos pos;
    pos.b = item / H;
    pos.h = item % H;
    pos.g = pos.h / HG;
    pos.r = pos.h % HG;
    auto step = [&](ItemPos q) {
        q.r += Sr;
        q.g += Sg;
        if (q.r >= HG) {
            q.r -= HG;
            ++q.g;
        }
        q.h += Sh;
        q.b += Sb;
        if (q.h >= H) {
            q.h -= H;
            ++q.b;
            q.g -= G;
        }
        return q;
    };

    // issue the copies of `it`'s chunks (at position q) into stage `s` (one commit group), and
    // return its x
    auto prefetch = [&](int it, const ItemPos& q, int s, float (&xq)[CH]) {
        const int b = q.b, g = q.g;
        const uint4* st = reinterpret_cast<const uint4*>(state_q + (size_t)it * P * N);
        const int8_t* xrow = x + (size_t)it * P;
#pragma unroll
        for (int k = 0; k < CH; ++k) {
            const int u = tid + k * TPB;
            const bool in = k * TPB < nchunks && u < nchunks;
            if (in) cp_async16(&sq[s][k][tid], st + u);
            xq[k] = in ? static_cast<float>(xrow[u / CPR]) : 0.f;
        }
        if (tid < 2 * CPR) {
            const int8_t* row = (tid < CPR ? Bq : Cq) + ((size_t)b * G + g) * N;
            cp_async16(&sbc[s][tid], row + 16 * (tid % CPR));
        }
        cp_async_commit();
    };

    float xq[CH], xq_n[CH];
    prefetch(item, pos, 0, xq);
    float dtv = dt[item], s_old = state_scale[item];
    for (int it = 0;; ++it) {
        const int s = it & 1;
        const int next = item + gridDim.x;
        const ItemPos npos = step(pos);
        float dt_n = 0.f, s_old_n = 0.f;
        if (next < count) {
            prefetch(next, npos, s ^ 1, xq_n);
            dt_n = dt[next];
            s_old_n = state_scale[next];
            cp_async_wait<1>();  // this item's group has landed (the next one may be in flight)
        } else {
            cp_async_wait<0>();
        }
        const int h = pos.h, g = pos.g;
        const float sx = x_scale[h], Dh = D[h];
        const float decay = __expf(dtv * A[h]);
        float4* sb = sbv[s];
        float4* sc = scv[s];
        if (tid < 2 * CPR) {
            f2 v[8];
            unpack16(sbc[s][tid], v);
            // scales per group, or per group and dstate channel (SSDi8 Table 10, per-P(N)):
            // this chunk holds channels 16 (tid % CPR) .. + 15
            const float* sp = tid < CPR ? B_scale : C_scale;
            float4* dst = (tid < CPR ? sb : sc) + tid % CPR;
            if (per_n) {
                const float* sv = sp + (size_t)g * N + 16 * (tid % CPR);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i * CPR] = make_float4(sv[4 * i] * v[2 * i].x, sv[4 * i + 1] * v[2 * i].y,
                                               sv[4 * i + 2] * v[2 * i + 1].x,
                                               sv[4 * i + 3] * v[2 * i + 1].y);
            } else {
                const float sv = sp[g];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i * CPR] = make_float4(sv * v[2 * i].x, sv * v[2 * i].y, sv * v[2 * i + 1].x, sv * v[2 * i + 1].y);
            }
        }
        __syncthreads();

        const f2 ds = {decay * s_old, decay * s_old};  // decayed dequantisation factor
        float amax = 0.f;
        // the loop bound is warp-uniform (multiples of the CTA size) so that every lane reaches
        // the shuffles
#pragma unroll
        for (int k = 0; k < CH; ++k) {
            if (k * TPB >= nchunks) break;
            const int u = tid + k * TPB;
            const bool in = u < nchunks;
            const int p = in ? u / CPR : 0, cc = u % CPR;
            // (a thread past the last chunk copied nothing: its zero codes keep the max clean)
            f2 hv[8];
            unpack16(in ? sq[s][k][tid] : make_uint4(0u, 0u, 0u, 0u), hv);
            const float xv = sx * xq[k];
            const f2 dx = {dtv * xv, dtv * xv};
            f2 acc = {0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 bb = sb[i * CPR + cc], cq = sc[i * CPR + cc];
                hv[2 * i] = ffma2(ds, hv[2 * i], fmul2(dx, f2{bb.x, bb.y}));
                hv[2 * i + 1] = ffma2(ds, hv[2 * i + 1], fmul2(dx, f2{bb.z, bb.w}));
                acc = ffma2(f2{cq.x, cq.y}, hv[2 * i], acc);
                acc = ffma2(f2{cq.z, cq.w}, hv[2 * i + 1], acc);
                amax = amax3(amax3(amax, hv[2 * i]), hv[2 * i + 1]);
            }
            float a = acc.x + acc.y;
#pragma unroll
            for (int o = CPR / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
            if (in && (lane % CPR) == 0) {
                if constexpr (HAD) ys[p] = a + Dh * xv;
                else store_out(y, (size_t)item * P + p, a + Dh * xv, y_dtype, inv_y_scale);
            }
        }
        amax = block_max<TPB>(amax, scratch);  // (its barrier also completes ys)
        if constexpr (HAD) {
            if (tid < kWarp) hadamard64_store(ys, y, (size_t)item * P, y_dtype, inv_y_scale);
        }
        const float inv = amax > 0.f ? 127.f / amax : 0.f;
        uint4* st = reinterpret_cast<uint4*>(state_q + (size_t)item * P * N);
#pragma unroll
        for (int k = 0; k < CH; ++k) {
            if (k * TPB >= nchunks) break;
            const int u = tid + k * TPB;
            if (u >= nchunks) continue;
            const int cc = u % CPR;
            const float xv = sx * xq[k];
            const f2 dx = {dtv * xv, dtv * xv};
            f2 hv[8];
            unpack16(sq[s][k][tid], hv);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 bb = sb[i * CPR + cc];
                hv[2 * i] = ffma2(ds, hv[2 * i], fmul2(dx, f2{bb.x, bb.y}));
                hv[2 * i + 1] = ffma2(ds, hv[2 * i + 1], fmul2(dx, f2{bb.z, bb.w}));
            }
            st[u] = pack16_fma(hv, inv);  // the same fp32 values as the max pass (same operations)
        }
        if (tid == 0) state_scale[item] = amax / 127.f;
        if (next >= count) break;
        item = next;
        pos = npos;
        dtv = dt_n;
        s_old = s_old_n;
#pragma unroll
        for (int k = 0; k < CH; ++k) xq[k] = xq_n[k];
    }
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

// Resident CTAs of state_update_q8_kernel<N, TPB, CH, HAD> on the current device (SMs x CTAs
// per SM), looked up once per device and instantiation.
template <int N, int TPB, int CH, bool HAD>
int resident_ctas() {
    constexpr int kMaxDevices = 64;
    static int cache[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    if (cache[dev] == 0) {
        int sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                &per_sm, state_update_q8_kernel<N, TPB, CH, HAD>, TPB, 0) != cudaSuccess)
            return 0;
        cache[dev] = sms * (per_sm > 0 ? per_sm : 1);
    }
    return cache[dev];
}

template <int N, bool HAD>
cudaError_t launch_q8_nh(const StateUpdateQ8Args& a, cudaStream_t st) {
    const int count = a.batch * a.nheads;
    return with_shape(a.headdim * N / 16, [&](auto tpb, auto ch) {
        constexpr int TPB = decltype(tpb)::value, CH = decltype(ch)::value;
        const int resident = resident_ctas<N, TPB, CH, HAD>();
        if (resident <= 0) return cudaErrorUnknown;
        const int grid = count < resident ? count : resident;
        state_update_q8_kernel<N, TPB, CH, HAD><<<grid, TPB, 0, st>>>(
            a.state_q, a.state_scale, a.x, a.B, a.C, a.dt, a.A, a.D, a.x_scale, a.B_scale,
            a.C_scale, count, a.nheads, a.headdim, a.ngroups, a.per_n, a.y, a.y_dtype,
            a.inv_y_scale);
        return cudaGetLastError();
    });
}

template <int N>
cudaError_t launch_q8_n(const StateUpdateQ8Args& a, cudaStream_t st) {
    return a.hadamard ? launch_q8_nh<N, true>(a, st) : launch_q8_nh<N, false>(a, st);
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
