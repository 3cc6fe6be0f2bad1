// Forward entry point that needs no caller-provided workspace.
//
// Who needs this: code that receives only its input and output buffers and is
// not allowed to allocate device memory itself, for example a plugin called from
// another framework's execution hook (that framework owns and has already
// reserved the device memory, so an extra cudaMalloc may fail or silently break
// its memory plan), or a latency-bound loop where cudaMalloc / cudaFree cannot
// be afforded because they synchronise the device. Such callers cannot provide
// the scratch workspace that dspark_attn_fwd asks for.
//
// What it does: it runs exactly the dspark_attn_fwd sequence, with the
// workspace placed in a fixed, file-scope device array compiled into this
// library instead of a caller buffer. The array is not allocated at run time:
// every GPU that loads the library holds it (DSPARK_NOALLOC_SCRATCH_BYTES)
// until the process exits.
#include <mutex>

#include "dspark_internal.cuh"

namespace {

constexpr size_t kScratchBytes = DSPARK_NOALLOC_SCRATCH_BYTES;

// The scratch workspace. In host code this name is only a stand-in for the
// device symbol, not a device address: the address is looked up per device
// with cudaGetSymbolAddress and passed to the kernels as an ordinary pointer.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device. Outside a
// stream capture it is looked up on every call (cudaGetSymbolAddress, with the
// device current), so that an address cached before a cudaDeviceReset (which
// reloads the module and may move the array) is never used again. While the
// stream is being captured the address cached by the last uncaptured call on
// this device is used; a capture before any uncaptured call on the device
// attempts the lookup as well.
dspark_status scratch_address(cudaStream_t st, void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSPARK_ERR_CUDA;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return DSPARK_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (cap == cudaStreamCaptureStatusNone || !g_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DSPARK_ERR_CUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return DSPARK_OK;
}

}  // namespace

extern "C" dspark_status dspark_attn_fwd_noalloc(const dspark_problem *p, const void *q, const void *kc,
                                                 const void *kr, const void *v, const int32_t *anchors,
                                                 const uint8_t *keep, void *o, float *lse, uint32_t *error_word,
                                                 void *stream) {
    const size_t need = dspark::fwd_workspace_size(p);  // the forward's part of the layout
    if (need == 0) {
        // invalid problem: the regular entry point reports the precise status
        // from its host-side checks, before any device work
        return dspark_attn_fwd(p, q, kc, kr, v, anchors, keep, o, lse, nullptr, 0, 0, stream);
    }
    if (need > kScratchBytes) return DSPARK_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    const dspark_status s0 = scratch_address((cudaStream_t)stream, &scratch);
    if (s0 != DSPARK_OK) return s0;
    // The descriptor is rebuilt on every call (which also clears the error
    // word); everything else the forward reads from the scratch is fully
    // rewritten before it is read, so the previous call's contents never leak.
    const dspark_status s = dspark_attn_fwd(p, q, kc, kr, v, anchors, keep, o, lse, scratch, kScratchBytes, 0, stream);
    if (s != DSPARK_OK) return s;
    if (error_word) {
        // the error word sits at offset 0 of the workspace layout
        if (cudaMemcpyAsync(error_word, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice, (cudaStream_t)stream) !=
            cudaSuccess)
            return DSPARK_ERR_CUDA;
    }
    return DSPARK_OK;
}
