// ssd_i8_chunk_scan_noalloc: the chunk scan for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run the scan: code executing
// under a fixed memory budget that was reserved up front (an inference engine that hands out
// every byte of its pool before serving), code that must not synchronise the device (a
// cudaMalloc can), and plug-ins of hosts that own all allocation.  For them this entry point
// takes the scan's scratch from a fixed array compiled into the library instead of a
// caller-provided workspace.  Everything else -- inputs, outputs, stream -- is the caller's, as
// for ssd_i8_chunk_scan, and the same kernels run.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds its
// kScratchBytes until the process exits.  In host code its name is only a host-side stand-in,
// so its device address is looked up once per device with cudaGetSymbolAddress (with that
// device current) and cached.
#include <cstdint>
#include <mutex>

#include "../../include/ssd_i8.h"

namespace {

// Built-in scratch: 4 MiB, the workspace of problems with up to 127 work items of 128 tokens,
// batch * nheads * ceil(seqlen / 128) <= 127 whatever the chunk size (the chunk scan hands
// states between CTAs through one 32 KiB slot per CTA, one CTA per work item at most).
constexpr size_t kScratchBytes = size_t(4) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device; looked up on the first call per device.
// With `lookup` false, a device whose address was never looked up (no call ran there) gives
// *out = nullptr.
ssd_status scratch_on_current_device(void** out, bool lookup = true) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return SSD_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SSD_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_ptr[dev] == nullptr && lookup) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return SSD_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return SSD_OK;
}

}  // namespace

extern "C" ssd_status ssd_i8_chunk_scan_noalloc(
    const int8_t* x, const int8_t* B, const int8_t* C, const float* dt, const float* A,
    const float* D, const float* x_scale, const float* B_scale, const float* C_scale, int batch,
    int seqlen, int nheads, int headdim, int dstate, int ngroups, int chunk_size,
    const float* init_state, float* final_state, void* y, int y_dtype, float y_scale,
    void* stream) {
    const size_t need = ssd_i8_chunk_scan_workspace_size(batch, seqlen, nheads, headdim, dstate,
                                                         ngroups, chunk_size);
    if (need > kScratchBytes) return SSD_ERR_WORKSPACE;  // problem too large for the built-in scratch
    void* scratch = nullptr;
    if (need > 0) {
        const ssd_status s = scratch_on_current_device(&scratch);
        if (s != SSD_OK) return s;
    }
    // Nothing in the scratch has to start at zero: the hand-off flags and the status word are
    // tagged with a per-call 64-bit epoch, so a previous call's leftovers never match, and a
    // state slot is read only after its flag carries this call's epoch.
    return ssd_i8_chunk_scan(x, B, C, dt, A, D, x_scale, B_scale, C_scale, batch, seqlen, nheads,
                             headdim, dstate, ngroups, chunk_size, init_state, final_state, y,
                             y_dtype, y_scale, scratch, kScratchBytes, stream);
}

// The kernel writes its failure words at the start of whatever scratch it ran on, so the
// workspace status query reads them from the built-in array as well.
extern "C" ssd_status ssd_i8_chunk_scan_noalloc_status(void* stream) {
    void* scratch = nullptr;
    const ssd_status s = scratch_on_current_device(&scratch, false);
    if (s != SSD_OK) return s;
    if (scratch == nullptr) {  // no allocation-free call has run on this device
        if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return SSD_ERR_CUDA;
        return SSD_OK;
    }
    return ssd_i8_chunk_scan_status(scratch, stream);
}
