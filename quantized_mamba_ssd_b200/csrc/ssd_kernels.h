// Internal launcher interface between the C ABI (abi.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace ssd {

struct ChunkScanArgs {
    const int8_t* x;
    const int8_t* B;
    const int8_t* C;
    const float* dt;
    const float* A;
    const float* D;
    const float* x_scale;
    const float* B_scale;
    const float* C_scale;
    int batch, seqlen, nheads, headdim, dstate, ngroups, chunk_size;
    const float* init_state;
    float* final_state;
    void* y;
    int y_dtype;  // SSD_OUT_* code with the SSD_OUT_HADAMARD / SSD_SCALES_PER_N flags
    float inv_y_scale;
    void* workspace;
    // packed variable-length sequences (seq_tab == null: `batch` contiguous rows of `seqlen`)
    const void* seq_tab;        // device: int4 {first token, tokens, block prefix, caller index}
    int nseq;                   // entries of seq_tab
    long long total_tokens;     // packed tokens addressed by x, B, C, dt, y
    long long total_blocks;     // sum over the table of ceil(tokens / 128)
    long long x_token_stride;   // bytes between consecutive tokens of x (heads contiguous)
    long long bc_token_stride;  // bytes between consecutive tokens of B and of C
    long long dt_token_stride;  // elements between consecutive tokens of dt
};

struct StateUpdateArgs {
    float* state;
    const int8_t* x;
    const int8_t* B;
    const int8_t* C;
    const float* dt;
    const float* A;
    const float* D;
    const float* x_scale;
    const float* B_scale;
    const float* C_scale;
    int batch, nheads, headdim, dstate, ngroups;
    void* y;
    int y_dtype;  // SSD_OUT_* without the Hadamard flag
    float inv_y_scale;
    int hadamard;  // 1: y' = H y / 8 over headdim (64) before the conversion
    int per_n;     // 1: B_scale / C_scale are [ngroups, dstate]
};

struct StateUpdateQ8Args {
    int8_t* state_q;     // [batch, nheads, headdim, dstate] codes
    float* state_scale;  // [batch, nheads]
    const int8_t* x;
    const int8_t* B;
    const int8_t* C;
    const float* dt;
    const float* A;
    const float* D;
    const float* x_scale;
    const float* B_scale;
    const float* C_scale;
    int batch, nheads, headdim, dstate, ngroups;
    void* y;
    int y_dtype;  // SSD_OUT_* without the Hadamard flag
    float inv_y_scale;
    int hadamard;  // 1: y' = H y / 8 over headdim (64) before the conversion
    int per_n;     // 1: B_scale / C_scale are [ngroups, dstate]
};

size_t chunk_scan_workspace_bytes(int batch, int seqlen, int nheads, int headdim, int dstate,
                                  int chunk_size);
// workspace of the variable-length scan: header, flags, 256 slots, then the sequence table
size_t chunk_scan_varlen_workspace_bytes(int nseq);
size_t chunk_scan_varlen_table_offset();
cudaError_t launch_chunk_scan(const ChunkScanArgs& a, cudaStream_t stream);
cudaError_t launch_chunk_cb(const int8_t* C, const int8_t* B, int batch, int seqlen, int ngroups,
                            int dstate, int chunk_size, int32_t* cb, cudaStream_t stream);
cudaError_t launch_state_update(const StateUpdateArgs& a, cudaStream_t stream);
bool state_q8_shape_ok(int headdim, int dstate);
cudaError_t launch_state_update_q8(const StateUpdateQ8Args& a, cudaStream_t stream);
cudaError_t launch_state_quantize(const float* state, int8_t* q, float* scale, int count,
                                  int headdim, int dstate, cudaStream_t stream);
void arm_fault_injection(int drop_publish_cta, long long wait_cycles);
// Epoch of the first chunk-scan launch on `workspace` since the last call of this function for
// it (false: none launched since); the entry is removed.
bool take_first_epoch(const void* workspace, unsigned long long* epoch);

}  // namespace ssd
