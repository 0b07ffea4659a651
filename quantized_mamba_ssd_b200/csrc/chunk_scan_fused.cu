// Fused int8 SSD chunk scan for sm_100a: one persistent CTA per SM, tcgen05 tensor cores,
// TMA-staged int8 tiles, the running state kept in tensor memory.
//
// Work: units u = (batch, head), each a sequence of nch = ceil(L / Q) chunks.  The flattened
// (unit, chunk) list is cut into one contiguous range per CTA, so every SM gets the same
// number of chunks.  A range holds at most one unit piece that starts mid-sequence (its first)
// and one that ends mid-sequence (its last).  The CTA runs its last piece first and publishes
// the state at its end to a workspace slot; it runs its first piece last, after reading the
// predecessor CTA's slot (a bounded wait).  With at least nch chunks per CTA the slot is
// always ready by then.
//
// Per chunk of Q tokens and one head (SSDi8 page: ChunkState, state path, ChunkScan,
// ChunkBMM of Table 5; X_scaled of Figure 3(a)):
//   Acum_t = sum_{k<=t} dt_k A_h                     block scan, fp32
//   CB     = Cq Bq^T                                  tcgen05 kind::i8, exact int32 in TMEM
//   M'     = CB * exp(Acum_t - Acum_s) * dt_s / kappa  (s <= t), f16, written over CB in TMEM
//   acc    = C' H'^T + M' x                           tcgen05 kind::f16, A from TMEM
//            C'[t,n] = Cq[t,n] exp(Acum_t),  H' = H / kappa
//   y      = s_C s_x s_B kappa acc + D s_x xq           fused epilogue (f32 / f16 / int8)
//   H     <- exp(Acum_end) H + B'^T x,  B'[t,n] = Bq[t,n] dt_t exp(Acum_end - Acum_t)
// H is kept in units of s_x s_B.  Only the operands that are not int8 (M', C', B', H') are
// rounded, once each, to f16 (relative 2^-12); kappa keeps them inside f16 range.
#include <algorithm>
#include <atomic>
#include <mutex>
#include <random>

#include "common.cuh"
#include "sm100.cuh"
#include "ssd_kernels.h"

namespace ssd {
namespace {

using namespace sm100;

constexpr int kThreads = 128;  // one warpgroup: thread i <-> TMEM lane i
constexpr int kP = 64;         // headdim
constexpr int kTB = 128;       // rows of a t-block (MMA M)
constexpr long long kWaitCycles = 1ll << 31;  // bound of every device-side wait (~1 s)
constexpr int kMaxCtas = 256;  // workspace slots

// tensor memory columns (512 allocated)
constexpr uint32_t kColCB = 0;     // 256: CB int32; M' f16 pairs written over it
constexpr uint32_t kColAcc = 256;  // 64: y accumulator f32 [t][p]
constexpr uint32_t kColC = 320;    // 64: C' f16 pairs [t][n]
constexpr uint32_t kColH = 384;    // 64: state f32 [n][p]
constexpr uint32_t kTmemCols = 512;

template <int Q>
struct Layout {
    static constexpr int kC = 0;                        // Cq  [Q][128 B], 128B swizzle
    static constexpr int kB = kC + Q * 128;             // Bq  [Q][128 B], 128B swizzle
    static constexpr int kXf = kB + Q * 128;            // x f16 [Q][64] (MN-major, swizzled)
    static constexpr int kBp = kXf + Q * 128;           // B' f16 2 x [Q][64] (MN-major)
    static constexpr int kHp = kBp + 2 * Q * 128;       // H' f16 [128 n][64 p] (MN-major)
    static constexpr int kX = kHp + 128 * 128;          // xq [Q][64 B], dense
    static constexpr int kDt = kX + Q * 64;             // dt [256] f32
    static constexpr int kAcum = kDt + 256 * 4;         // Acum [256] f32
    static constexpr int kRed = kAcum + 256 * 4;        // reduction scratch [64] f32
    static constexpr int kBar = kRed + 64 * 4;          // 4 mbarriers
    static constexpr int kMisc = kBar + 4 * 8;          // tmem base, abort flag
    static constexpr int kBytes = kMisc + 16;
    static constexpr int kAlloc = kBytes + 1024;        // + alignment slack
    static_assert(kXf % 1024 == 0 && kBp % 1024 == 0 && kHp % 1024 == 0 && kB % 1024 == 0,
                  "swizzled tiles must be 1024-byte aligned");
};

struct FusedParams {
    const float* dt;
    const float* A;
    const float* D;
    const float* x_scale;
    const float* B_scale;
    const float* C_scale;
    const float* init_state;
    float* final_state;
    void* y;
    int y_dtype;
    float inv_y_scale;
    int batch, L, H, G, N, nch, nctas;
    long long total;  // batch * H * nch
    float* slots;     // [nctas][128 n][64 p] handed-off states (units of s_x s_B)
    unsigned long long* flags;   // [nctas] epoch of the published slot
    unsigned long long* status;  // [3]: epoch and code of a device-side failure, last epoch
    unsigned long long epoch;
};

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

// int8x4 (one 32-bit word) -> 4 floats
__device__ __forceinline__ void i8x4_to_f32(uint32_t w, float* f) {
    f[0] = static_cast<float>(static_cast<int8_t>(w & 0xff));
    f[1] = static_cast<float>(static_cast<int8_t>((w >> 8) & 0xff));
    f[2] = static_cast<float>(static_cast<int8_t>((w >> 16) & 0xff));
    f[3] = static_cast<float>(static_cast<int8_t>(w >> 24));
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x / 32;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[warp] = v;
    __syncthreads();
    return fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
}

__device__ void report_failure(const FusedParams& p, unsigned long long code) {
    p.status[1] = code;
    __threadfence();
    atomicExch(p.status, p.epoch);
}

// Issue the ChunkBMM MMAs: D[tmem] = C rows [t0, t0+128) x B rows [0, ncols), K = 128 (int8).
__device__ __forceinline__ void issue_cb(uint32_t d, uint32_t sC, uint32_t sB, int t0, int ncols) {
    const uint32_t id = idesc_i8(kTB, ncols, false, false);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint64_t a = smem_desc(sC + t0 * 128 + 32 * k, 16, 1024, kSwizzle128B);
        const uint64_t b = smem_desc(sB + 32 * k, 16, 1024, kSwizzle128B);
        mma_i8_ss(d, a, b, id, k > 0);
    }
}

template <int Q>
__global__ void __launch_bounds__(kThreads, 1)
fused_chunk_scan_kernel(const __grid_constant__ CUtensorMap map_x,
                        const __grid_constant__ CUtensorMap map_B,
                        const __grid_constant__ CUtensorMap map_C, const FusedParams p) {
    using Lay = Layout<Q>;
    constexpr int NTB = Q > kTB ? Q / kTB : 1;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sC = smem + Lay::kC;
    uint8_t* sB = smem + Lay::kB;
    uint8_t* sXf = smem + Lay::kXf;
    uint8_t* sBp = smem + Lay::kBp;
    uint8_t* sHp = smem + Lay::kHp;
    const uint8_t* sX = smem + Lay::kX;
    float* dts = reinterpret_cast<float*>(smem + Lay::kDt);
    float* acum = reinterpret_cast<float*>(smem + Lay::kAcum);
    float* red = reinterpret_cast<float*>(smem + Lay::kRed);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBar);
    uint64_t* bar_tma = bars + 0;
    uint64_t* bar_cb = bars + 1;
    uint64_t* bar_acc = bars + 2;
    uint64_t* bar_state = bars + 3;
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::kMisc);
    volatile uint32_t* abort_flag = misc + 1;

    const int tid = threadIdx.x;
    const int warp = tid / 32;
    const uint32_t lane_base = static_cast<uint32_t>(warp) * 32u;

    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(bars + i, 1);
        fence_mbar_init();
        *abort_flag = 0;
        if (blockIdx.x == 0) p.status[2] = p.epoch;  // the call the status word refers to
        tma_prefetch_map(&map_x);
        tma_prefetch_map(&map_B);
        tma_prefetch_map(&map_C);
    }
    if (warp == 0) {
        tmem_alloc(misc, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    uint32_t ph_tma = 0, ph_cb = 0, ph_acc = 0, ph_state = 0;
    bool tma_in_flight = false;

    // wait helper: every thread waits; a timeout raises the CTA-wide abort flag
    auto wait_bar = [&](uint64_t* bar, uint32_t& phase) {
        if (!mbar_wait(bar, phase, kWaitCycles)) *abort_flag = 1;
        phase ^= 1u;
    };

    const long long W = p.total;
    const int cta = blockIdx.x;
    const long long ws = W * cta / p.nctas, we = W * (cta + 1) / p.nctas;
    const int nch = p.nch;
    const long long u_first = ws / nch, u_last = (we - 1) / nch;
    const int nseg = we > ws ? static_cast<int>(u_last - u_first + 1) : 0;

    for (int k = 0; k < nseg && !*abort_flag; ++k) {
        const long long u = (k == 0) ? u_last : (k == nseg - 1 ? u_first : u_first + k);
        const int c_begin = static_cast<int>(u == u_first ? ws - u * nch : 0);
        const int c_end = static_cast<int>(u == u_last ? we - u * nch : nch);
        const int b = static_cast<int>(u / p.H), h = static_cast<int>(u % p.H);
        const int g = h / (p.H / p.G);
        const float sx = p.x_scale[h], sBg = p.B_scale[g], sCg = p.C_scale[g];
        const float sigma = sx * sBg;
        const float A_h = p.A[h], Dsx = p.D[h] * sx;
        const int N = p.N;
        const int n = tid;  // state row owned by this thread (TMEM lane)

        // ---- initial state of the piece -> H (TMEM lanes = n, columns = p) ----
        {
            const float* src = nullptr;
            float scale = 1.f / sigma;
            if (c_begin == 0) {
                if (p.init_state) src = p.init_state + ((size_t)b * p.H + h) * kP * N;
            } else {
                if (tid == 0) {
                    const unsigned long long* f = p.flags + (cta - 1);
                    const long long t0 = clock64();
                    unsigned long long v;
                    for (;;) {
                        asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(f) : "memory");
                        if (v == p.epoch) break;
                        if (clock64() - t0 > kWaitCycles) {
                            report_failure(p, 2);
                            *abort_flag = 1;
                            break;
                        }
                        __nanosleep(256);
                    }
                }
                __syncthreads();
                if (*abort_flag) break;
                src = p.slots + (size_t)(cta - 1) * 128 * kP;
                scale = 1.f;
            }
            uint32_t r[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int pp = half * 32 + j;
                    float v = 0.f;
                    if (src != nullptr && n < N)
                        v = (c_begin == 0) ? src[(size_t)pp * N + n] * scale : __ldcg(src + n * kP + pp);
                    r[j] = __float_as_uint(v);
                }
                tmem_st32(tmem_addr(tmem, lane_base, kColH + half * 32), r);
            }
            tmem_st_wait();
        }

        for (int c = c_begin; c < c_end; ++c) {
            const int t_base = c * Q;
            const int valid = min(Q, p.L - t_base);
            // ---- TMA: x, B, C tiles of the chunk (zero past the sequence end) ----
            if (tid == 0) {
                mbar_arrive_expect_tx(bar_tma, Q * 128 * 2 + Q * 64);
                tma_load_4d(smem + Lay::kX, &map_x, 0, h, t_base, b, bar_tma);
                tma_load_4d(sB, &map_B, 0, g, t_base, b, bar_tma);
                tma_load_4d(sC, &map_C, 0, g, t_base, b, bar_tma);
            }
            tma_in_flight = true;
            // ---- chunk_cumsum: Acum_t (inclusive), two tokens per thread ----
            float dmax;
            {
                const int t0 = 2 * tid, t1 = 2 * tid + 1;
                const float* dtp = p.dt + ((size_t)b * p.L + t_base) * p.H + h;
                const float d0 = (t0 < valid) ? dtp[(size_t)t0 * p.H] : 0.f;
                const float d1 = (t1 < valid) ? dtp[(size_t)t1 * p.H] : 0.f;
                const float a0 = d0 * A_h, a1 = d1 * A_h;
                const float incl = block_inclusive_scan(a0 + a1, red);
                const float excl = incl - (a0 + a1);
                if (t0 < Q) {
                    dts[t0] = d0;
                    acum[t0] = excl + a0;
                }
                if (t1 < Q) {
                    dts[t1] = d1;
                    acum[t1] = excl + a0 + a1;
                }
                dmax = block_max(fmaxf(d0, d1), red + 32);
            }
            __syncthreads();
            const float a_end = acum[Q - 1];
            const float decay_end = __expf(a_end);

            // ---- chunk boundary: H' = f16(H / kappa) for C'.H', then H <- exp(Acum_end) H ----
            float kappa;
            {
                uint32_t hv[2][32];
                tmem_ld32(tmem_addr(tmem, lane_base, kColH), hv[0]);
                tmem_ld32(tmem_addr(tmem, lane_base, kColH + 32), hv[1]);
                tmem_ld_wait();
                float m = 0.f;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(__uint_as_float(hv[hh][j])));
                const float hmax = block_max(m, red + 40);
                kappa = fmaxf(hmax, 16129.f * static_cast<float>(N) * dmax) * (1.f / 16384.f);
                if (!(kappa > 1e-30f) || !isfinite(kappa)) kappa = 1.f;
                const float inv_k = 1.f / kappa;
                // H' row n: 64 f16 = 128 bytes, 8 swizzled 16-byte chunks
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const int hh = ch / 4, j0 = (ch % 4) * 8;
                    uint4 v;
                    v.x = pack_f16x2(__uint_as_float(hv[hh][j0 + 0]) * inv_k, __uint_as_float(hv[hh][j0 + 1]) * inv_k);
                    v.y = pack_f16x2(__uint_as_float(hv[hh][j0 + 2]) * inv_k, __uint_as_float(hv[hh][j0 + 3]) * inv_k);
                    v.z = pack_f16x2(__uint_as_float(hv[hh][j0 + 4]) * inv_k, __uint_as_float(hv[hh][j0 + 5]) * inv_k);
                    v.w = pack_f16x2(__uint_as_float(hv[hh][j0 + 6]) * inv_k, __uint_as_float(hv[hh][j0 + 7]) * inv_k);
                    *reinterpret_cast<uint4*>(sHp + sw128(n, ch * 16)) = v;
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        hv[hh][j] = __float_as_uint(__uint_as_float(hv[hh][j]) * decay_end);
                    tmem_st32(tmem_addr(tmem, lane_base, kColH + hh * 32), hv[hh]);
                }
                tmem_st_wait();
            }

            // ---- wait for the tiles, then convert x -> f16 and B -> B' (f16) ----
            wait_bar(bar_tma, ph_tma);
            tma_in_flight = false;
            for (int t = tid; t < Q; t += kThreads) {
                // x row t: 64 int8 (dense) -> 64 f16 (swizzled 128-byte row)
                const uint4* xs = reinterpret_cast<const uint4*>(sX + t * 64);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint4 w = xs[q4];
                    const uint32_t ws4[4] = {w.x, w.y, w.z, w.w};
                    float f[16];
#pragma unroll
                    for (int i = 0; i < 4; ++i) i8x4_to_f32(ws4[i], f + 4 * i);
                    uint4 o0, o1;
                    o0.x = pack_f16x2(f[0], f[1]);   o0.y = pack_f16x2(f[2], f[3]);
                    o0.z = pack_f16x2(f[4], f[5]);   o0.w = pack_f16x2(f[6], f[7]);
                    o1.x = pack_f16x2(f[8], f[9]);   o1.y = pack_f16x2(f[10], f[11]);
                    o1.z = pack_f16x2(f[12], f[13]); o1.w = pack_f16x2(f[14], f[15]);
                    *reinterpret_cast<uint4*>(sXf + sw128(t, q4 * 32)) = o0;
                    *reinterpret_cast<uint4*>(sXf + sw128(t, q4 * 32 + 16)) = o1;
                }
                // B row t (128-byte swizzled int8) scaled by w_t -> B' (two 64-column blocks)
                const float w_t = (t < valid) ? dts[t] * __expf(a_end - acum[t]) : 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint4 w = *reinterpret_cast<const uint4*>(sB + sw128(t, j * 16));
                    const uint32_t ws4[4] = {w.x, w.y, w.z, w.w};
                    float f[16];
#pragma unroll
                    for (int i = 0; i < 4; ++i) i8x4_to_f32(ws4[i], f + 4 * i);
                    uint4 o0, o1;
                    o0.x = pack_f16x2(f[0] * w_t, f[1] * w_t);   o0.y = pack_f16x2(f[2] * w_t, f[3] * w_t);
                    o0.z = pack_f16x2(f[4] * w_t, f[5] * w_t);   o0.w = pack_f16x2(f[6] * w_t, f[7] * w_t);
                    o1.x = pack_f16x2(f[8] * w_t, f[9] * w_t);   o1.y = pack_f16x2(f[10] * w_t, f[11] * w_t);
                    o1.z = pack_f16x2(f[12] * w_t, f[13] * w_t); o1.w = pack_f16x2(f[14] * w_t, f[15] * w_t);
                    uint8_t* blk = sBp + (j / 4) * (Q * 128);
                    *reinterpret_cast<uint4*>(blk + sw128(t, (j % 4) * 32)) = o0;
                    *reinterpret_cast<uint4*>(blk + sw128(t, (j % 4) * 32 + 16)) = o1;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            if (*abort_flag) break;

            // ---- state update MMA: H += B'^T x  (M = 128 n, N = 64 p, K = Q) ----
            if (tid == 0) {
                const uint32_t id = idesc_f16(128, kP, true, true);
#pragma unroll 4
                for (int kk = 0; kk < Q / 16; ++kk) {
                    const uint64_t a = smem_desc(smem_u32(sBp) + 2048 * kk, Q * 128, 1024, kSwizzle128B);
                    const uint64_t bd = smem_desc(smem_u32(sXf) + 2048 * kk, 16, 1024, kSwizzle128B);
                    mma_f16_ss(tmem + kColH, a, bd, id, 1);
                }
                tc_commit(bar_state);
            }

            // ---- t-blocks of 128 rows ----
            const float rho = sCg * sigma * kappa;
            const float inv_kappa = 1.f / kappa;
            for (int tb = 0; tb < NTB; ++tb) {
                const int t0 = tb * kTB;
                const int ncols = (Q <= kTB) ? Q : (tb + 1) * kTB;
                const int t = t0 + tid;  // this thread's row
                // C' row t -> TMEM (64 columns of f16 pairs); rows past Q are zero
                {
                    const float f = (t < Q) ? __expf(acum[t]) : 0.f;
                    uint32_t r[32];
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
#pragma unroll
                        for (int j4 = 0; j4 < 4; ++j4) {
                            const int j = half * 4 + j4;  // 16-byte chunk of the int8 row
                            uint4 w = make_uint4(0, 0, 0, 0);
                            if (t < Q) w = *reinterpret_cast<const uint4*>(sC + sw128(t, j * 16));
                            const uint32_t ws4[4] = {w.x, w.y, w.z, w.w};
                            float fv[16];
#pragma unroll
                            for (int i = 0; i < 4; ++i) i8x4_to_f32(ws4[i], fv + 4 * i);
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                r[j4 * 8 + i] = pack_f16x2(fv[2 * i] * f, fv[2 * i + 1] * f);
                        }
                        tmem_st32(tmem_addr(tmem, lane_base, kColC + half * 32), r);
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                __syncthreads();
                tc_fence_after();
                if (tid == 0) {
                    issue_cb(tmem + kColCB, smem_u32(sC), smem_u32(sB), t0, ncols);
                    tc_commit(bar_cb);
                    const uint32_t id = idesc_f16(kTB, kP, false, true);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_f16_ts(tmem + kColAcc, tmem + kColC + 8 * kk,
                                   smem_desc(smem_u32(sHp) + 2048 * kk, 16, 1024, kSwizzle128B), id,
                                   kk > 0);
                }
                wait_bar(bar_cb, ph_cb);
                tc_fence_after();
                // M' over CB, in place: columns [32 sc, 32 sc + 32) -> f16 pairs at [16 sc, 16 sc + 16)
                {
                    const float at = (t < Q) ? acum[t] : 0.f;
                    const bool row_ok = t < valid;
                    for (int sc = 0; sc < ncols / 32; ++sc) {
                        uint32_t r[32];
                        tmem_ld32(tmem_addr(tmem, lane_base, kColCB + 32 * sc), r);
                        tmem_ld_wait();
                        uint32_t o[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float mv[2];
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int s = 32 * sc + 2 * i + e;
                                float v = 0.f;
                                if (row_ok && s <= t)
                                    v = static_cast<float>(static_cast<int>(r[2 * i + e])) *
                                        __expf(at - acum[s]) * dts[s] * inv_kappa;
                                mv[e] = v;
                            }
                            o[i] = pack_f16x2(mv[0], mv[1]);
                        }
                        tmem_st16(tmem_addr(tmem, lane_base, kColCB + 16 * sc), o);
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                __syncthreads();
                tc_fence_after();
                if (*abort_flag) break;
                if (tid == 0) {
                    const uint32_t id = idesc_f16(kTB, kP, false, true);
                    for (int kk = 0; kk < ncols / 16; ++kk)
                        mma_f16_ts(tmem + kColAcc, tmem + kColCB + 8 * kk,
                                   smem_desc(smem_u32(sXf) + 2048 * kk, 16, 1024, kSwizzle128B), id,
                                   1);
                    tc_commit(bar_acc);
                }
                wait_bar(bar_acc, ph_acc);
                tc_fence_after();
                // ---- epilogue: y = rho * acc + D s_x xq ----
                {
                    uint32_t r[2][32];
                    tmem_ld32(tmem_addr(tmem, lane_base, kColAcc), r[0]);
                    tmem_ld32(tmem_addr(tmem, lane_base, kColAcc + 32), r[1]);
                    tmem_ld_wait();
                    if (t < valid) {
                        const size_t ybase = (((size_t)b * p.L + t_base + t) * p.H + h) * kP;
                        const int8_t* xr = reinterpret_cast<const int8_t*>(sX + t * 64);
                        float out[kP];
#pragma unroll
                        for (int pp = 0; pp < kP; ++pp)
                            out[pp] = rho * __uint_as_float(r[pp / 32][pp % 32]) +
                                      Dsx * static_cast<float>(xr[pp]);
                        if (p.y_dtype == SSD_OUT_I8) {
                            int8_t* yo = static_cast<int8_t*>(p.y) + ybase;
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                uint32_t wv[4];
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    uint32_t acc = 0;
#pragma unroll
                                    for (int e = 0; e < 4; ++e) {
                                        float rr = rintf(out[q * 16 + i * 4 + e] * p.inv_y_scale);
                                        rr = fminf(fmaxf(rr, -127.f), 127.f);
                                        acc |= (static_cast<uint32_t>(static_cast<int>(rr)) & 0xffu) << (8 * e);
                                    }
                                    wv[i] = acc;
                                }
                                reinterpret_cast<uint4*>(yo)[q] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                            }
                        } else if (p.y_dtype == SSD_OUT_F16) {
                            __half* yo = static_cast<__half*>(p.y) + ybase;
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                reinterpret_cast<uint4*>(yo)[q] = make_uint4(
                                    pack_f16x2(out[q * 8 + 0], out[q * 8 + 1]), pack_f16x2(out[q * 8 + 2], out[q * 8 + 3]),
                                    pack_f16x2(out[q * 8 + 4], out[q * 8 + 5]), pack_f16x2(out[q * 8 + 6], out[q * 8 + 7]));
                        } else {
                            float* yo = static_cast<float*>(p.y) + ybase;
#pragma unroll
                            for (int q = 0; q < 16; ++q)
                                reinterpret_cast<float4*>(yo)[q] =
                                    make_float4(out[q * 4], out[q * 4 + 1], out[q * 4 + 2], out[q * 4 + 3]);
                        }
                    }
                }
                tc_fence_before();
                __syncthreads();
                tc_fence_after();
            }
            // the state MMA of this chunk must be done before the next boundary step reads H
            wait_bar(bar_state, ph_state);
            tc_fence_after();
            __syncthreads();
            if (*abort_flag) break;
        }
        if (*abort_flag) break;

        // ---- end of the piece: final state and / or hand-off slot ----
        {
            uint32_t hv[2][32];
            tmem_ld32(tmem_addr(tmem, lane_base, kColH), hv[0]);
            tmem_ld32(tmem_addr(tmem, lane_base, kColH + 32), hv[1]);
            tmem_ld_wait();
            if (c_end == nch) {
                if (p.final_state != nullptr && n < N) {
                    float* dst = p.final_state + ((size_t)b * p.H + h) * kP * N;
#pragma unroll
                    for (int pp = 0; pp < kP; ++pp)
                        dst[(size_t)pp * N + n] = sigma * __uint_as_float(hv[pp / 32][pp % 32]);
                }
            } else {
                float4* dst = reinterpret_cast<float4*>(p.slots + ((size_t)cta * 128 + n) * kP);
#pragma unroll
                for (int q = 0; q < kP / 4; ++q)
                    dst[q] = make_float4(__uint_as_float(hv[(4 * q) / 32][(4 * q) % 32]),
                                         __uint_as_float(hv[(4 * q + 1) / 32][(4 * q + 1) % 32]),
                                         __uint_as_float(hv[(4 * q + 2) / 32][(4 * q + 2) % 32]),
                                         __uint_as_float(hv[(4 * q + 3) / 32][(4 * q + 3) % 32]));
                __threadfence();
                __syncthreads();
                if (tid == 0) {
                    unsigned long long* f = p.flags + cta;
                    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(f), "l"(p.epoch) : "memory");
                }
            }
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
        }
    }

    // ---- teardown: nothing of ours may still be in flight when TMEM is released ----
    if (*abort_flag) {
        if (tid == 0) report_failure(p, 1);
        if (tma_in_flight) mbar_wait(bar_tma, ph_tma, kWaitCycles);
        if (tid == 0) tc_commit(bar_acc);
        mbar_wait(bar_acc, ph_acc, kWaitCycles);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ChunkBMM export with the same device code the fused scan uses: one CTA per
// (chunk, group, batch), t-blocks of 128 rows, every s column of the chunk.
template <int Q>
__global__ void __launch_bounds__(kThreads, 1)
chunk_cb_tc_kernel(const __grid_constant__ CUtensorMap map_B, const __grid_constant__ CUtensorMap map_C,
                   int nch, int G, int32_t* __restrict__ cb) {
    constexpr int NTB = Q > kTB ? Q / kTB : 1;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sC = smem;
    uint8_t* sB = smem + Q * 128;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * Q * 128);
    uint32_t* misc = reinterpret_cast<uint32_t*>(bars + 2);
    const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid / 32;
    if (tid == 0) {
        mbar_init(bars, 1);
        mbar_init(bars + 1, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(misc, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    if (tid == 0) {
        mbar_arrive_expect_tx(bars, Q * 128 * 2);
        tma_load_4d(sB, &map_B, 0, g, c * Q, b, bars);
        tma_load_4d(sC, &map_C, 0, g, c * Q, b, bars);
    }
    bool ok = mbar_wait(bars, 0, kWaitCycles);
    uint32_t ph = 0;
    int32_t* out = cb + (((size_t)b * nch + c) * G + g) * Q * Q;
    for (int tb = 0; tb < NTB && ok; ++tb) {
        if (tid == 0) {
            issue_cb(tmem, smem_u32(sC), smem_u32(sB), tb * kTB, Q);
            tc_commit(bars + 1);
        }
        ok = mbar_wait(bars + 1, ph, kWaitCycles);
        ph ^= 1u;
        tc_fence_after();
        const int t = tb * kTB + tid;
        for (int sc = 0; sc < Q / 32; ++sc) {
            uint32_t r[32];
            tmem_ld32(tmem_addr(tmem, warp * 32, 32 * sc), r);
            tmem_ld_wait();
            if (t < Q) {
#pragma unroll
                for (int j = 0; j < 32; ++j) out[(size_t)t * Q + 32 * sc + j] = static_cast<int32_t>(r[j]);
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// 4-D int8 map over [batch][L][rows2][inner] with box {box0, 1, Q, 1}.
bool make_map(CUtensorMap* m, const void* base, int inner, int rows2, int L, int batch, int box0,
              int Q, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)rows2, (cuuint64_t)L, (cuuint64_t)batch};
    cuuint64_t strides[3] = {(cuuint64_t)inner, (cuuint64_t)inner * rows2,
                             (cuuint64_t)inner * rows2 * L};
    cuuint32_t box[4] = {(cuuint32_t)box0, 1, (cuuint32_t)Q, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

std::atomic<unsigned long long>& epoch_counter() {
    static std::atomic<unsigned long long> ctr{[] {
        std::random_device rd;
        return (static_cast<unsigned long long>(rd()) << 32) ^ rd() ^ 0x5bd1e995ull;
    }()};
    return ctr;
}

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

template <int Q>
cudaError_t launch_fused_q(const ChunkScanArgs& a, cudaStream_t st) {
    CUtensorMap mx, mB, mC;
    if (!make_map(&mx, a.x, kP, a.nheads, a.seqlen, a.batch, kP, Q, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&mB, a.B, a.dstate, a.ngroups, a.seqlen, a.batch, 128, Q, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mC, a.C, a.dstate, a.ngroups, a.seqlen, a.batch, 128, Q, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    FusedParams p{};
    p.dt = a.dt; p.A = a.A; p.D = a.D; p.x_scale = a.x_scale; p.B_scale = a.B_scale;
    p.C_scale = a.C_scale; p.init_state = a.init_state; p.final_state = a.final_state;
    p.y = a.y; p.y_dtype = a.y_dtype; p.inv_y_scale = a.inv_y_scale;
    p.batch = a.batch; p.L = a.seqlen; p.H = a.nheads; p.G = a.ngroups; p.N = a.dstate;
    p.nch = ceil_div(a.seqlen, Q);
    p.total = (long long)a.batch * a.nheads * p.nch;
    int sms = num_sms();
    if (sms <= 0) return cudaErrorInvalidDevice;
    long long nctas = std::min<long long>(std::min(sms, kMaxCtas), p.total);
    p.nctas = static_cast<int>(nctas);
    uint8_t* ws = static_cast<uint8_t*>(a.workspace);
    p.status = reinterpret_cast<unsigned long long*>(ws);
    p.flags = reinterpret_cast<unsigned long long*>(ws + 256);
    p.slots = reinterpret_cast<float*>(ws + 256 + kMaxCtas * 8);
    p.epoch = ++epoch_counter();
    // at least 120 KB of shared memory per CTA keeps it alone on its SM: the kernel takes all of
    // the SM's tensor memory and CTAs wait on their predecessor's hand-off
    const int smem = std::max(Layout<Q>::kAlloc, 120 * 1024);
    cudaError_t e = cudaFuncSetAttribute(fused_chunk_scan_kernel<Q>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    fused_chunk_scan_kernel<Q><<<p.nctas, kThreads, smem, st>>>(mx, mB, mC, p);
    return cudaGetLastError();
}

template <int Q>
cudaError_t launch_cb_q(const int8_t* C, const int8_t* B, int batch, int seqlen, int G, int N,
                        int32_t* cb, cudaStream_t st) {
    CUtensorMap mB, mC;
    if (!make_map(&mB, B, N, G, seqlen, batch, 128, Q, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mC, C, N, G, seqlen, batch, 128, Q, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int nch = ceil_div(seqlen, Q);
    const int smem = 2 * Q * 128 + 64 + 1024;
    cudaError_t e = cudaFuncSetAttribute(chunk_cb_tc_kernel<Q>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(nch, G, batch);
    chunk_cb_tc_kernel<Q><<<grid, kThreads, smem, st>>>(mB, mC, nch, G, cb);
    return cudaGetLastError();
}

}  // namespace

size_t chunk_scan_workspace_bytes(int batch, int seqlen, int nheads, int headdim, int dstate,
                                  int chunk_size) {
    (void)headdim;
    (void)dstate;
    const long long total = (long long)batch * nheads * ceil_div(seqlen, chunk_size);
    const long long slots = std::min<long long>(total, kMaxCtas);
    return 256 + kMaxCtas * 8 + (size_t)slots * 128 * kP * 4;
}

cudaError_t launch_chunk_scan(const ChunkScanArgs& a, cudaStream_t st) {
    switch (a.chunk_size) {
        case 64: return launch_fused_q<64>(a, st);
        case 128: return launch_fused_q<128>(a, st);
        case 256: return launch_fused_q<256>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_chunk_cb(const int8_t* C, const int8_t* B, int batch, int seqlen, int G,
                            int N, int Q, int32_t* cb, cudaStream_t st) {
    switch (Q) {
        case 64: return launch_cb_q<64>(C, B, batch, seqlen, G, N, cb, st);
        case 128: return launch_cb_q<128>(C, B, batch, seqlen, G, N, cb, st);
        case 256: return launch_cb_q<256>(C, B, batch, seqlen, G, N, cb, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ssd
