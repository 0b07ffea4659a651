// extern "C" entry points of libssd_i8.so: argument checks, then one launch sequence on the
// caller's stream.  Declarations and their documentation live in include/ssd_i8.h.
#include <cmath>
#include <cstdint>
#include <vector>

#include "../../include/ssd_i8.h"
#include "ssd_kernels.h"

namespace {

constexpr int kAbiVersion = 1;
constexpr size_t kWorkspaceAlign = 256;

bool valid_out_dtype(int d) { return d == SSD_OUT_F32 || d == SSD_OUT_F16 || d == SSD_OUT_I8; }

// chunk-scan and decode outputs may also carry the Hadamard and per-channel-scale flags
bool valid_scan_out(int d) { return valid_out_dtype(d & ~(SSD_OUT_HADAMARD | SSD_SCALES_PER_N)); }

bool chunk_dstate_ok(int n) { return n == 16 || n == 32 || n == 64 || n == 128; }

bool chunk_size_ok(int q) { return q == 64 || q == 128 || q == 256; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Output scale handling shared by both entry points: I8 needs y_scale > 0 (finite); the
// kernels multiply by its fp32 reciprocal.
bool out_scale(int y_dtype, float y_scale, float* inv) {
    *inv = 1.f;
    if ((y_dtype & ~(SSD_OUT_HADAMARD | SSD_SCALES_PER_N)) != SSD_OUT_I8) return true;
    if (!(y_scale > 0.f) || !std::isfinite(y_scale)) return false;
    *inv = 1.f / y_scale;
    return std::isfinite(*inv);
}

}  // namespace

extern "C" {

int ssd_i8_abi_version(void) { return kAbiVersion; }

const char* ssd_status_string(ssd_status s) {
    switch (s) {
        case SSD_OK: return "SSD_OK";
        case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG: invalid argument";
        case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: shape not supported by the kernels";
        case SSD_ERR_WORKSPACE: return "SSD_ERR_WORKSPACE: workspace missing, too small or misaligned";
        case SSD_ERR_CUDA: return "SSD_ERR_CUDA: CUDA runtime or launch failure";
        case SSD_ERR_TIMEOUT: return "SSD_ERR_TIMEOUT: a bounded device-side wait gave up";
        default: return "SSD_ERR_UNKNOWN";
    }
}

size_t ssd_i8_chunk_scan_workspace_size(int batch, int seqlen, int nheads, int headdim,
                                        int dstate, int ngroups, int chunk_size) {
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0 ||
        chunk_size <= 0)
        return 0;
    const size_t n = ssd::chunk_scan_workspace_bytes(batch, seqlen, nheads, headdim, dstate,
                                                     chunk_size);
    return (n + kWorkspaceAlign - 1) / kWorkspaceAlign * kWorkspaceAlign;
}

ssd_status ssd_i8_chunk_scan(const int8_t* x, const int8_t* B, const int8_t* C, const float* dt,
                             const float* A, const float* D, const float* x_scale,
                             const float* B_scale, const float* C_scale, int batch, int seqlen,
                             int nheads, int headdim, int dstate, int ngroups, int chunk_size,
                             const float* init_state, float* final_state, void* y, int y_dtype,
                             float y_scale, void* workspace, size_t workspace_bytes,
                             void* stream) {
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0 ||
        chunk_size <= 0 || nheads % ngroups != 0 || !valid_scan_out(y_dtype))
        return SSD_ERR_INVALID_ARG;
    if (!A || !D || !x_scale || !B_scale || !C_scale) return SSD_ERR_INVALID_ARG;
    if (headdim != 64 || !chunk_dstate_ok(dstate) || !chunk_size_ok(chunk_size))
        return SSD_ERR_UNSUPPORTED;
    // the kernel indexes (sequence, head) units with 32-bit integers
    if ((long long)batch * nheads > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;
    float inv = 1.f;
    if (!out_scale(y_dtype, y_scale, &inv)) return SSD_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t state_bytes = (size_t)batch * nheads * headdim * dstate * sizeof(float);
    if (batch == 0) return SSD_OK;
    if (seqlen == 0) {
        // nothing to scan: the final state is the initial state
        if (final_state) {
            cudaError_t e = init_state ? cudaMemcpyAsync(final_state, init_state, state_bytes,
                                                         cudaMemcpyDeviceToDevice, st)
                                       : cudaMemsetAsync(final_state, 0, state_bytes, st);
            if (e != cudaSuccess) return SSD_ERR_CUDA;
        }
        return SSD_OK;
    }
    if (!x || !B || !C || !dt || !y) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(B) || !aligned16(C) || !aligned16(y)) return SSD_ERR_INVALID_ARG;
    const size_t need = ssd_i8_chunk_scan_workspace_size(batch, seqlen, nheads, headdim, dstate,
                                                         ngroups, chunk_size);
    if (!workspace || workspace_bytes < need ||
        reinterpret_cast<uintptr_t>(workspace) % kWorkspaceAlign != 0)
        return SSD_ERR_WORKSPACE;
    ssd::ChunkScanArgs a{x, B, C, dt, A, D, x_scale, B_scale, C_scale, batch, seqlen, nheads,
                         headdim, dstate, ngroups, chunk_size, init_state, final_state, y,
                         y_dtype, inv, workspace};
    return ssd::launch_chunk_scan(a, st) == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

size_t ssd_i8_chunk_scan_varlen_workspace_size(int nseq) {
    if (nseq < 0) return 0;
    const size_t n = ssd::chunk_scan_varlen_workspace_bytes(nseq);
    return (n + kWorkspaceAlign - 1) / kWorkspaceAlign * kWorkspaceAlign;
}

ssd_status ssd_i8_chunk_scan_varlen(const int8_t* x, long long x_token_stride, const int8_t* B,
                                    const int8_t* C, long long bc_token_stride, const float* dt,
                                    long long dt_token_stride, const float* A, const float* D,
                                    const float* x_scale, const float* B_scale,
                                    const float* C_scale, const int32_t* cu_seqlens, int nseq,
                                    long long total_tokens, int nheads, int headdim, int dstate,
                                    int ngroups, int chunk_size, const float* init_state,
                                    float* final_state, void* y, int y_dtype, float y_scale,
                                    void* workspace, size_t workspace_bytes, void* stream) {
    if (nseq < 0 || total_tokens < 0 || total_tokens > 0x7fffffffLL || nheads <= 0 ||
        headdim <= 0 || dstate <= 0 || ngroups <= 0 || chunk_size <= 0 ||
        nheads % ngroups != 0 || !valid_scan_out(y_dtype) || !cu_seqlens)
        return SSD_ERR_INVALID_ARG;
    if (!A || !D || !x_scale || !B_scale || !C_scale) return SSD_ERR_INVALID_ARG;
    if (headdim != 64 || !chunk_dstate_ok(dstate) || !chunk_size_ok(chunk_size))
        return SSD_ERR_UNSUPPORTED;
    float inv = 1.f;
    if (!out_scale(y_dtype, y_scale, &inv)) return SSD_ERR_INVALID_ARG;
    // sequences: non-decreasing offsets inside [0, total_tokens]
    if (nseq > 0 && (cu_seqlens[0] < 0 || cu_seqlens[nseq] > total_tokens)) return SSD_ERR_INVALID_ARG;
    for (int s = 0; s < nseq; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return SSD_ERR_INVALID_ARG;
    // strides: TMA needs 16-byte multiples; rows must not overlap
    if (x_token_stride < (long long)nheads * headdim || x_token_stride % 16 != 0 ||
        bc_token_stride < (long long)ngroups * dstate || bc_token_stride % 16 != 0 ||
        dt_token_stride < nheads)
        return SSD_ERR_INVALID_ARG;
    if (nseq == 0) return SSD_OK;
    const size_t need = ssd_i8_chunk_scan_varlen_workspace_size(nseq);
    if (!workspace || workspace_bytes < need ||
        reinterpret_cast<uintptr_t>(workspace) % kWorkspaceAlign != 0)
        return SSD_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t state_elems = (size_t)nheads * headdim * dstate;
    // the table of non-empty sequences; an empty one only passes its initial state on
    std::vector<int32_t> tab;
    tab.reserve((size_t)nseq * 4);
    long long blocks = 0;
    for (int s = 0; s < nseq; ++s) {
        const int len = cu_seqlens[s + 1] - cu_seqlens[s];
        if (len == 0) {
            if (final_state) {
                float* dst = final_state + (size_t)s * state_elems;
                const cudaError_t e =
                    init_state ? cudaMemcpyAsync(dst, init_state + (size_t)s * state_elems,
                                                 state_elems * sizeof(float),
                                                 cudaMemcpyDeviceToDevice, st)
                               : cudaMemsetAsync(dst, 0, state_elems * sizeof(float), st);
                if (e != cudaSuccess) return SSD_ERR_CUDA;
            }
            continue;
        }
        tab.push_back(cu_seqlens[s]);
        tab.push_back(len);
        tab.push_back(static_cast<int32_t>(blocks));
        tab.push_back(s);
        blocks += (len + 127) / 128;
    }
    if (tab.empty()) return SSD_OK;
    if (blocks > 0x7fffffffLL || (long long)(tab.size() / 4) * nheads > 0x7fffffffLL)
        return SSD_ERR_UNSUPPORTED;
    if (!x || !B || !C || !dt || !y) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(B) || !aligned16(C) || !aligned16(y)) return SSD_ERR_INVALID_ARG;
    uint8_t* table = static_cast<uint8_t*>(workspace) + ssd::chunk_scan_varlen_table_offset();
    // pageable source: the copy is staged before the call returns, so `tab` may go away
    if (cudaMemcpyAsync(table, tab.data(), tab.size() * sizeof(int32_t), cudaMemcpyHostToDevice,
                        st) != cudaSuccess)
        return SSD_ERR_CUDA;
    ssd::ChunkScanArgs a{x, B, C, dt, A, D, x_scale, B_scale, C_scale, 0, 0, nheads,
                         headdim, dstate, ngroups, chunk_size, init_state, final_state, y,
                         y_dtype, inv, workspace};
    a.seq_tab = table;
    a.nseq = static_cast<int>(tab.size() / 4);
    a.total_tokens = total_tokens;
    a.total_blocks = blocks;
    a.x_token_stride = x_token_stride;
    a.bc_token_stride = bc_token_stride;
    a.dt_token_stride = dt_token_stride;
    return ssd::launch_chunk_scan(a, st) == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status ssd_i8_state_update(float* state, const int8_t* x, const int8_t* B, const int8_t* C,
                               const float* dt, const float* A, const float* D,
                               const float* x_scale, const float* B_scale, const float* C_scale,
                               int batch, int nheads, int headdim, int dstate, int ngroups,
                               void* y, int y_dtype, float y_scale, void* stream) {
    if (batch < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0 ||
        nheads % ngroups != 0 || !valid_scan_out(y_dtype))
        return SSD_ERR_INVALID_ARG;
    if (!(dstate == 16 || dstate == 32 || dstate == 64 || dstate == 128 || dstate == 256) ||
        headdim > 256 || ((y_dtype & SSD_OUT_HADAMARD) && headdim != 64))
        return SSD_ERR_UNSUPPORTED;
    float inv = 1.f;
    if (!out_scale(y_dtype, y_scale, &inv)) return SSD_ERR_INVALID_ARG;
    if (batch == 0) return SSD_OK;
    if (!state || !x || !B || !C || !dt || !A || !D || !x_scale || !B_scale || !C_scale || !y)
        return SSD_ERR_INVALID_ARG;
    ssd::StateUpdateArgs a{state, x, B, C, dt, A, D, x_scale, B_scale, C_scale, batch, nheads,
                           headdim, dstate, ngroups, y,
                           y_dtype & ~(SSD_OUT_HADAMARD | SSD_SCALES_PER_N), inv,
                           (y_dtype & SSD_OUT_HADAMARD) ? 1 : 0,
                           (y_dtype & SSD_SCALES_PER_N) ? 1 : 0};
    return ssd::launch_state_update(a, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SSD_OK
               : SSD_ERR_CUDA;
}

ssd_status ssd_i8_state_quantize(const float* state, int8_t* state_q, float* state_scale,
                                 int batch, int nheads, int headdim, int dstate, void* stream) {
    if (batch < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0) return SSD_ERR_INVALID_ARG;
    if (!ssd::state_q8_shape_ok(headdim, dstate)) return SSD_ERR_UNSUPPORTED;
    if (batch == 0) return SSD_OK;
    if (!state || !state_q || !state_scale) return SSD_ERR_INVALID_ARG;
    if (!aligned16(state) || !aligned16(state_q)) return SSD_ERR_INVALID_ARG;
    return ssd::launch_state_quantize(state, state_q, state_scale, batch * nheads, headdim, dstate,
                                      static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SSD_OK
               : SSD_ERR_CUDA;
}

ssd_status ssd_i8_state_update_q8(int8_t* state_q, float* state_scale, const int8_t* x,
                                  const int8_t* B, const int8_t* C, const float* dt,
                                  const float* A, const float* D, const float* x_scale,
                                  const float* B_scale, const float* C_scale, int batch,
                                  int nheads, int headdim, int dstate, int ngroups, void* y,
                                  int y_dtype, float y_scale, void* stream) {
    if (batch < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0 ||
        nheads % ngroups != 0 || !valid_scan_out(y_dtype))
        return SSD_ERR_INVALID_ARG;
    if (!ssd::state_q8_shape_ok(headdim, dstate) ||
        ((y_dtype & SSD_OUT_HADAMARD) && headdim != 64))
        return SSD_ERR_UNSUPPORTED;
    float inv = 1.f;
    if (!out_scale(y_dtype, y_scale, &inv)) return SSD_ERR_INVALID_ARG;
    if (batch == 0) return SSD_OK;
    if (!state_q || !state_scale || !x || !B || !C || !dt || !A || !D || !x_scale || !B_scale ||
        !C_scale || !y)
        return SSD_ERR_INVALID_ARG;
    if (!aligned16(state_q) || !aligned16(B) || !aligned16(C)) return SSD_ERR_INVALID_ARG;
    ssd::StateUpdateQ8Args a{state_q, state_scale, x, B, C, dt, A, D, x_scale, B_scale,
                             C_scale, batch, nheads, headdim, dstate, ngroups, y,
                             y_dtype & ~(SSD_OUT_HADAMARD | SSD_SCALES_PER_N), inv,
                             (y_dtype & SSD_OUT_HADAMARD) ? 1 : 0,
                             (y_dtype & SSD_SCALES_PER_N) ? 1 : 0};
    return ssd::launch_state_update_q8(a, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SSD_OK
               : SSD_ERR_CUDA;
}

ssd_status ssd_i8_chunk_cb(const int8_t* C, const int8_t* B, int batch, int seqlen, int ngroups,
                           int dstate, int chunk_size, int32_t* cb, void* stream) {
    if (batch < 0 || seqlen < 0 || ngroups <= 0 || dstate <= 0 || chunk_size <= 0)
        return SSD_ERR_INVALID_ARG;
    if (!chunk_dstate_ok(dstate) || !chunk_size_ok(chunk_size)) return SSD_ERR_UNSUPPORTED;
    if (batch == 0 || seqlen == 0) return SSD_OK;
    if (!C || !B || !cb) return SSD_ERR_INVALID_ARG;
    if (!aligned16(C) || !aligned16(B)) return SSD_ERR_INVALID_ARG;
    return ssd::launch_chunk_cb(C, B, batch, seqlen, ngroups, dstate, chunk_size, cb,
                                static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SSD_OK
               : SSD_ERR_CUDA;
}

ssd_status ssd_i8_debug_inject(int drop_publish_cta, long long wait_cycles) {
    if (drop_publish_cta < -1) return SSD_ERR_INVALID_ARG;
    ssd::arm_fault_injection(drop_publish_cta, wait_cycles);
    return SSD_OK;
}

ssd_status ssd_i8_chunk_scan_status(const void* workspace, void* stream) {
    if (!workspace) return SSD_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return SSD_ERR_CUDA;
    unsigned long long w[3] = {0, 0, 0};
    if (cudaMemcpy(w, workspace, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess)
        return SSD_ERR_CUDA;
    // w[0]: epoch of the last call that recorded a failure, w[1]: failure code, w[2]: epoch of
    // the last call that ran on this workspace.  Epochs grow by one per launch in a process, so
    // the calls since the previous query are those from `first` to w[2].
    unsigned long long first = 0;
    const bool since = ssd::take_first_epoch(workspace, &first);
    if (w[1] != 0 && (since ? (w[0] >= first && w[0] <= w[2]) : w[0] == w[2]))
        return SSD_ERR_TIMEOUT;
    return SSD_OK;
}

}  // extern "C"
