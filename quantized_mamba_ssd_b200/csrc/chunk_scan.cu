// Chunked int8 SSD scan: chunk_cumsum + chunk_state, state passing, chunk_scan.
//
// The decomposition of the scan into chunks of Q tokens (SSDi8 page, Figure 1(b) and the
// ChunkState / ChunkBMM modules of Table 5):
//
//   Acum_t   = sum_{k <= t, k in chunk} dt_k A_h                      (chunk_cumsum)
//   S_c      = sum_{t in c} w_t x_t B_t^T,  w_t = dt_t exp(Acum_end - Acum_t)
//              (the decay folded into x: SSDi8's X_scaled = X * LUT_state, Figure 3(a))
//   H_c      = exp(Acum_end,c) H_{c-1} + S_c                          (state passing)
//   y_t      = s_x s_B s_C sum_{s<=t} CB[t,s] exp(Acum_t - Acum_s) dt_s xq_s
//              + s_C exp(Acum_t) Cq_t H_{c-1} + D s_x xq_t             (chunk_scan)
//   CB[t,s]  = sum_n Cq[t,n] Bq[s,n]   exact int32 (ChunkBMM on the int8 codes)
//
// This file is the CUDA-core version: three kernels with the chunk states in the workspace.
#include "common.cuh"
#include "ssd_kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kP = 64;  // headdim supported by these kernels

// ---------------------------------------------------------------------------------------
// per-chunk prefix sums of dt*A (chunk_cumsum), into smem arrays acum[] and dts[]
// ---------------------------------------------------------------------------------------
__device__ void chunk_cumsum(const float* __restrict__ dt, float A_h, int b, int c, int h,
                             int L, int H, int Q, float* dts, float* acum, float* scan_scratch) {
    const int t = threadIdx.x;  // blockDim.x >= Q
    const int l = c * Q + t;
    float d = 0.f;
    if (t < Q && l < L) d = dt[((size_t)b * L + l) * H + h];
    float v = block_inclusive_scan(d * A_h, scan_scratch);
    if (t < Q) {
        dts[t] = d;
        acum[t] = v;
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------------------
// Kernel 1: chunk states S_c[p, n] (fp32) and the chunk decay totals Acum_end.
// grid (nchunks, H, batch), block 256.
// ---------------------------------------------------------------------------------------
template <int N>
__global__ void __launch_bounds__(kThreads)
chunk_state_kernel(const int8_t* __restrict__ x, const int8_t* __restrict__ Bq,
                   const float* __restrict__ dt, const float* __restrict__ A,
                   const float* __restrict__ x_scale, const float* __restrict__ B_scale,
                   int L, int H, int G, int Q, float* __restrict__ states,
                   float* __restrict__ dA_end) {
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int nchunks = gridDim.x;
    const int g = h / (H / G);
    extern __shared__ __align__(16) unsigned char smem[];
    float* dts = reinterpret_cast<float*>(smem);          // [Q]
    float* acum = dts + 256;                               // [Q]
    float* w = acum + 256;                                 // [Q]
    float* scratch = w + 256;                              // [32]
    int8_t* xs = reinterpret_cast<int8_t*>(scratch + 32);  // [Q][P]
    int8_t* bs = xs + 256 * kP;                            // [Q][N]

    chunk_cumsum(dt, A[h], b, c, h, L, H, Q, dts, acum, scratch);
    const int valid = min(Q, L - c * Q);
    const float a_end = acum[valid - 1];
    for (int t = threadIdx.x; t < Q; t += kThreads)
        w[t] = t < valid ? dts[t] * __expf(a_end - acum[t]) : 0.f;
    // stage x and B rows of the chunk (16-byte vectors), zero past the sequence end
    for (int i = threadIdx.x; i < Q * kP / 16; i += kThreads) {
        const int t = i / (kP / 16), v = i % (kP / 16);
        int4 val = make_int4(0, 0, 0, 0);
        if (t < valid)
            val = reinterpret_cast<const int4*>(x + (((size_t)b * L + c * Q + t) * H + h) * kP)[v];
        reinterpret_cast<int4*>(xs)[i] = val;
    }
    for (int i = threadIdx.x; i < Q * N / 16; i += kThreads) {
        const int t = i / (N / 16), v = i % (N / 16);
        int4 val = make_int4(0, 0, 0, 0);
        if (t < valid)
            val = reinterpret_cast<const int4*>(Bq + (((size_t)b * L + c * Q + t) * G + g) * N)[v];
        reinterpret_cast<int4*>(bs)[i] = val;
    }
    __syncthreads();

    // thread -> (p, n-block): p = tid % 64, n in [nb * N/4, (nb + 1) * N/4)
    constexpr int NPT = N / 4;
    const int p = threadIdx.x % kP, nb = threadIdx.x / kP;
    float acc[NPT];
#pragma unroll
    for (int j = 0; j < NPT; ++j) acc[j] = 0.f;
    for (int t = 0; t < valid; ++t) {
        const float xv = w[t] * static_cast<float>(xs[t * kP + p]);
        const int8_t* brow = bs + t * N + nb * NPT;
#pragma unroll
        for (int j = 0; j < NPT; ++j) acc[j] = fmaf(xv, static_cast<float>(brow[j]), acc[j]);
    }
    const float sc = x_scale[h] * B_scale[g];
    float* out = states + ((((size_t)b * nchunks + c) * H + h) * kP + p) * N + nb * NPT;
#pragma unroll
    for (int j = 0; j < NPT; j += 4)
        *reinterpret_cast<float4*>(out + j) =
            make_float4(acc[j] * sc, acc[j + 1] * sc, acc[j + 2] * sc, acc[j + 3] * sc);
    if (threadIdx.x == 0) dA_end[((size_t)b * nchunks + c) * H + h] = a_end;
}

// ---------------------------------------------------------------------------------------
// Kernel 2: state passing H_c = exp(Acum_end,c) H_{c-1} + S_c, sequential over chunks.
// Overwrites states[c] with the state ENTERING chunk c.  grid (ceil(P*N/256), H, batch).
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads)
state_passing_kernel(float* __restrict__ states, const float* __restrict__ dA_end,
                     const float* __restrict__ init_state, float* __restrict__ final_state,
                     int nchunks, int H, int PN) {
    const int e = blockIdx.x * kThreads + threadIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    if (e >= PN) return;
    float hs = init_state ? init_state[((size_t)b * H + h) * PN + e] : 0.f;
    const size_t stride = (size_t)H * PN;
    float* s = states + ((size_t)b * nchunks * H + h) * PN + e;
    const float* da = dA_end + (size_t)b * nchunks * H + h;
    float next = nchunks > 0 ? s[0] : 0.f;
    for (int c = 0; c < nchunks; ++c) {
        const float cur = next;
        if (c + 1 < nchunks) next = s[(size_t)(c + 1) * stride];
        s[(size_t)c * stride] = hs;
        hs = __expf(da[(size_t)c * H]) * hs + cur;
    }
    if (final_state) final_state[((size_t)b * H + h) * PN + e] = hs;
}

// ---------------------------------------------------------------------------------------
// CB tile rows: cb[i][s] for rows t0..t0+rows-1 and columns s < ncols of one chunk/group.
// ---------------------------------------------------------------------------------------
template <int N>
__device__ __forceinline__ int cb_entry(const int8_t* crow, const int8_t* brow) {
    const int* c4 = reinterpret_cast<const int*>(crow);
    const int* b4 = reinterpret_cast<const int*>(brow);
    int acc = 0;
#pragma unroll
    for (int k = 0; k < N / 4; ++k) acc = dot4_i8(c4[k], b4[k], acc);
    return acc;
}

// ---------------------------------------------------------------------------------------
// Kernel 3: chunk_scan with the fused output epilogue.  grid (nchunks, H, batch).
// ---------------------------------------------------------------------------------------
constexpr int kRows = 16;  // output rows (tokens) per pass

template <int N>
__global__ void __launch_bounds__(kThreads)
chunk_scan_kernel(const int8_t* __restrict__ x, const int8_t* __restrict__ Bq,
                  const int8_t* __restrict__ Cq, const float* __restrict__ dt,
                  const float* __restrict__ A, const float* __restrict__ D,
                  const float* __restrict__ x_scale, const float* __restrict__ B_scale,
                  const float* __restrict__ C_scale, int L, int H, int G, int Q,
                  const float* __restrict__ states, void* __restrict__ y, int y_dtype,
                  float inv_y_scale) {
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int nchunks = gridDim.x;
    const int g = h / (H / G);
    constexpr int HP = N + 1;  // padded row pitch of the state tile (bank-conflict free)
    extern __shared__ __align__(16) unsigned char smem[];
    float* dts = reinterpret_cast<float*>(smem);          // [256]
    float* acum = dts + 256;                               // [256]
    float* scratch = acum + 256;                           // [32]
    float* hs = scratch + 32;                              // [P][N+1]
    float* m = hs + kP * HP;                               // [kRows][256]
    int8_t* xs = reinterpret_cast<int8_t*>(m + kRows * 256);  // [Q][P]
    int8_t* bs = xs + 256 * kP;                            // [Q][N]
    int8_t* cs = bs + 256 * N;                             // [Q][N]

    chunk_cumsum(dt, A[h], b, c, h, L, H, Q, dts, acum, scratch);
    const int valid = min(Q, L - c * Q);
    for (int i = threadIdx.x; i < Q * kP / 16; i += kThreads) {
        const int t = i / (kP / 16), v = i % (kP / 16);
        int4 val = make_int4(0, 0, 0, 0);
        if (t < valid)
            val = reinterpret_cast<const int4*>(x + (((size_t)b * L + c * Q + t) * H + h) * kP)[v];
        reinterpret_cast<int4*>(xs)[i] = val;
    }
    for (int i = threadIdx.x; i < Q * N / 16; i += kThreads) {
        const int t = i / (N / 16), v = i % (N / 16);
        int4 vb = make_int4(0, 0, 0, 0), vc = make_int4(0, 0, 0, 0);
        if (t < valid) {
            const size_t off = (((size_t)b * L + c * Q + t) * G + g) * N;
            vb = reinterpret_cast<const int4*>(Bq + off)[v];
            vc = reinterpret_cast<const int4*>(Cq + off)[v];
        }
        reinterpret_cast<int4*>(bs)[i] = vb;
        reinterpret_cast<int4*>(cs)[i] = vc;
    }
    const float* hsrc = states + (((size_t)b * nchunks + c) * H + h) * kP * N;
    for (int i = threadIdx.x; i < kP * N; i += kThreads) hs[(i / N) * HP + (i % N)] = hsrc[i];
    __syncthreads();

    const float sx = x_scale[h], sB = B_scale[g], sC = C_scale[g], Dh = D[h];
    const float s_intra = sx * sB * sC;
    // thread -> (row i, p-group pg): p in {pg, pg+16, pg+32, pg+48}
    const int i_row = threadIdx.x / 16, pg = threadIdx.x % 16;
    for (int t0 = 0; t0 < valid; t0 += kRows) {
        const int rows = min(kRows, valid - t0);
        const int scols = t0 + rows;  // causal: columns s < t0 + rows
        // M[i][s] = CB[t][s] exp(Acum_t - Acum_s) dt_s for s <= t (else 0)
        for (int e = threadIdx.x; e < kRows * scols; e += kThreads) {
            const int i = e / scols, s = e % scols;
            const int t = t0 + i;
            float mv = 0.f;
            if (i < rows && s <= t) {
                const int cbv = cb_entry<N>(cs + t * N, bs + s * N);
                mv = static_cast<float>(cbv) * __expf(acum[t] - acum[s]) * dts[s];
            }
            m[i * 256 + s] = mv;
        }
        __syncthreads();
        if (i_row < rows) {
            const int t = t0 + i_row;
            float intra[4] = {0.f, 0.f, 0.f, 0.f}, inter[4] = {0.f, 0.f, 0.f, 0.f};
            for (int s = 0; s <= t; ++s) {
                const float mv = m[i_row * 256 + s];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    intra[j] = fmaf(mv, static_cast<float>(xs[s * kP + pg + 16 * j]), intra[j]);
            }
            const int8_t* crow = cs + t * N;
            for (int n = 0; n < N; ++n) {
                const float cv = static_cast<float>(crow[n]);
#pragma unroll
                for (int j = 0; j < 4; ++j) inter[j] = fmaf(cv, hs[(pg + 16 * j) * HP + n], inter[j]);
            }
            const float dec = sC * __expf(acum[t]);
            const size_t ybase = (((size_t)b * L + c * Q + t) * H + h) * kP;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int p = pg + 16 * j;
                const float xv = sx * static_cast<float>(xs[t * kP + p]);
                const float v = s_intra * intra[j] + dec * inter[j] + Dh * xv;
                store_out(y, ybase + p, v, y_dtype, inv_y_scale);
            }
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------------------
// ChunkBMM export: full Q x Q int32 blocks.  grid (nchunks, G, batch).
// ---------------------------------------------------------------------------------------
template <int N>
__global__ void __launch_bounds__(kThreads)
chunk_cb_kernel(const int8_t* __restrict__ Cq, const int8_t* __restrict__ Bq, int L, int G, int Q,
                int32_t* __restrict__ cb) {
    const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int nchunks = gridDim.x;
    extern __shared__ __align__(16) unsigned char smem[];
    int8_t* bs = reinterpret_cast<int8_t*>(smem);  // [Q][N]
    int8_t* cs = bs + 256 * N;                     // [Q][N]
    const int valid = min(Q, L - c * Q);
    for (int i = threadIdx.x; i < Q * N / 16; i += kThreads) {
        const int t = i / (N / 16), v = i % (N / 16);
        int4 vb = make_int4(0, 0, 0, 0), vc = make_int4(0, 0, 0, 0);
        if (t < valid) {
            const size_t off = (((size_t)b * L + c * Q + t) * G + g) * N;
            vb = reinterpret_cast<const int4*>(Bq + off)[v];
            vc = reinterpret_cast<const int4*>(Cq + off)[v];
        }
        reinterpret_cast<int4*>(bs)[i] = vb;
        reinterpret_cast<int4*>(cs)[i] = vc;
    }
    __syncthreads();
    int32_t* out = cb + (((size_t)b * nchunks + c) * G + g) * Q * Q;
    for (int e = threadIdx.x; e < Q * Q; e += kThreads) {
        const int t = e / Q, s = e % Q;
        out[e] = cb_entry<N>(cs + t * N, bs + s * N);
    }
}

template <int N>
cudaError_t launch_chunk_scan_n(const ChunkScanArgs& a, cudaStream_t st) {
    const int nchunks = ceil_div(a.seqlen, a.chunk_size);
    float* states = static_cast<float*>(a.workspace);
    float* dA = states + (size_t)a.batch * nchunks * a.nheads * kP * N;
    dim3 grid(nchunks, a.nheads, a.batch);
    const size_t smem1 = (3 * 256 + 32) * sizeof(float) + 256 * kP + 256 * N;
    cudaError_t e = cudaFuncSetAttribute(chunk_state_kernel<N>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
    if (e != cudaSuccess) return e;
    chunk_state_kernel<N><<<grid, kThreads, smem1, st>>>(a.x, a.B, a.dt, a.A, a.x_scale,
                                                         a.B_scale, a.seqlen, a.nheads,
                                                         a.ngroups, a.chunk_size, states, dA);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    dim3 g2(ceil_div(kP * N, kThreads), a.nheads, a.batch);
    state_passing_kernel<<<g2, kThreads, 0, st>>>(states, dA, a.init_state, a.final_state, nchunks,
                                                  a.nheads, kP * N);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t smem3 = (2 * 256 + 32 + kP * (N + 1) + kRows * 256) * sizeof(float) + 256 * kP +
                         2 * 256 * N;
    e = cudaFuncSetAttribute(chunk_scan_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem3);
    if (e != cudaSuccess) return e;
    chunk_scan_kernel<N><<<grid, kThreads, smem3, st>>>(
        a.x, a.B, a.C, a.dt, a.A, a.D, a.x_scale, a.B_scale, a.C_scale, a.seqlen, a.nheads,
        a.ngroups, a.chunk_size, states, a.y, a.y_dtype, a.inv_y_scale);
    return cudaGetLastError();
}

template <int N>
cudaError_t launch_chunk_cb_n(const int8_t* C, const int8_t* B, int batch, int seqlen, int G,
                              int Q, int32_t* cb, cudaStream_t st) {
    const int nchunks = ceil_div(seqlen, Q);
    dim3 grid(nchunks, G, batch);
    const size_t smem = 2 * 256 * N;
    cudaError_t e = cudaFuncSetAttribute(chunk_cb_kernel<N>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    chunk_cb_kernel<N><<<grid, kThreads, smem, st>>>(C, B, seqlen, G, Q, cb);
    return cudaGetLastError();
}

}  // namespace

size_t chunk_scan_workspace_bytes(int batch, int seqlen, int nheads, int headdim, int dstate,
                                  int chunk_size) {
    const size_t nchunks = (size_t)ceil_div(seqlen, chunk_size);
    const size_t states = (size_t)batch * nchunks * nheads * headdim * dstate * sizeof(float);
    const size_t da = (size_t)batch * nchunks * nheads * sizeof(float);
    return states + da;
}

cudaError_t launch_chunk_scan(const ChunkScanArgs& a, cudaStream_t st) {
    switch (a.dstate) {
        case 16: return launch_chunk_scan_n<16>(a, st);
        case 32: return launch_chunk_scan_n<32>(a, st);
        case 64: return launch_chunk_scan_n<64>(a, st);
        case 128: return launch_chunk_scan_n<128>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_chunk_cb(const int8_t* C, const int8_t* B, int batch, int seqlen, int ngroups,
                            int dstate, int chunk_size, int32_t* cb, cudaStream_t st) {
    switch (dstate) {
        case 16: return launch_chunk_cb_n<16>(C, B, batch, seqlen, ngroups, chunk_size, cb, st);
        case 32: return launch_chunk_cb_n<32>(C, B, batch, seqlen, ngroups, chunk_size, cb, st);
        case 64: return launch_chunk_cb_n<64>(C, B, batch, seqlen, ngroups, chunk_size, cb, st);
        case 128: return launch_chunk_cb_n<128>(C, B, batch, seqlen, ngroups, chunk_size, cb, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ssd
