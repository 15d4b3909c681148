// moba_attn_fwd_noalloc: the forward for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand the library a workspace buffer: plugin hosts
// that own every device allocation themselves, or services that forbid allocation once they
// have started.  For them this entry point runs the same forward as moba_attn_fwd, but its
// scratch lives in a fixed-size array in static device memory that belongs to the library.
//
// Costs and rules, stated once here and in include/moba.h:
//   - The array (MOBA_NOALLOC_SCRATCH_BYTES) is held on every GPU that loads the library,
//     until the process exits.
//   - The query-wave size is chosen per call so that the whole workspace fits the array;
//     a problem whose fixed part (block table, means, selections, routing lists) plus one
//     128-token wave does not fit is rejected with MOBA_ERR_UNSUPPORTED before any launch.
//   - Every call on a device shares the one array, and it keeps the last call's contents.
//     The forward re-initialises every field it reads (block table, status word, list
//     counters, work cursor) at the start of each call and wave.  Calls whose work overlaps
//     on the GPU (different streams, or different host threads) race on the array.
//   - The first call on each device looks up the array's device address with
//     cudaGetSymbolAddress while that device is current, and the address is kept for the
//     life of the process; that first call should come before any stream capture, and
//     destroying the device's primary context (cudaDeviceReset) invalidates the kept address.
//   - The forward's status word (MOBA_ERR_DEVICE_TIMEOUT when a bounded device wait gives up)
//     lives in the array; moba_device_status_noalloc reads it from the kept address.
//   - The call allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "moba.h"
#include "moba_internal.cuh"

namespace moba {
void set_error_message(const char* msg);
}

namespace {

__device__ __align__(256) static unsigned char g_scratch[MOBA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_setup_mutex;

// Largest multiple of 128 query tokens per wave whose workspace fits the array (0 = none).
int fitting_wave(moba_params pp) {
    const int T = pp.total_tokens;
    pp.wave_tokens = 0;
    const size_t whole = moba_workspace_size(&pp);
    if (whole != 0 && whole <= MOBA_NOALLOC_SCRATCH_BYTES &&
        (long long)T * pp.num_q_heads * pp.topk < 0x7fffffffLL)
        return 0;  // the whole input in one wave
    int lo = 0, hi = (T + 127) / 128;  // in units of 128 tokens
    while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        pp.wave_tokens = 128 * mid;
        const size_t need = moba_workspace_size(&pp);
        if (need != 0 && need <= MOBA_NOALLOC_SCRATCH_BYTES) lo = mid; else hi = mid - 1;
    }
    return 128 * lo;  // 0 when even one 128-token wave does not fit
}

// Kept scratch address of the current device, or nullptr when this process has not run an
// allocation-free forward there.  Sets *dev.
cudaError_t kept_scratch(int* dev, void** ptr) {
    *ptr = nullptr;
    const cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return e;
    if (*dev < 0 || *dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    *ptr = g_scratch_ptr[*dev];
    return cudaSuccess;
}

}  // namespace

extern "C" moba_status moba_device_status_noalloc(void* stream) {
    int dev = 0;
    void* scratch = nullptr;
    cudaError_t e = kept_scratch(&dev, &scratch);
    if (e != cudaSuccess) {
        moba::set_error_message(cudaGetErrorString(e));
        return MOBA_ERR_CUDA;
    }
    if (!scratch) return MOBA_OK;  // no allocation-free forward ran on this device
    // the workspace header sits at the start of the array
    const moba::WsHeader* hdr = static_cast<const moba::WsHeader*>(scratch);
    int word = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    e = cudaMemcpyAsync(&word, &hdr->status, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
        moba::set_error_message(cudaGetErrorString(e));
        return MOBA_ERR_CUDA;
    }
    if (word == 0) return MOBA_OK;
    char msg[64];
    snprintf(msg, sizeof(msg), "device status word %d", word);
    moba::set_error_message(msg);
    return (moba_status)word;
}

extern "C" moba_status moba_attn_fwd_noalloc(const moba_params* p, const void* q, const void* k,
                                            const void* v, const int* cu_seqlens, void* out,
                                            float* lse, void* stream) {
    if (!p) return moba_attn_fwd(p, q, k, v, cu_seqlens, nullptr, nullptr, nullptr, 0, out, lse,
                                 nullptr, stream);
    moba_params pp = *p;
    pp.wave_tokens = 0;
    if (moba_workspace_size(&pp) == 0 || pp.total_tokens == 0)
        // invalid parameters (reported by moba_attn_fwd's own checks) or nothing to do
        return moba_attn_fwd(&pp, q, k, v, cu_seqlens, nullptr, nullptr, nullptr, 0, out, lse,
                             nullptr, stream);
    const int wave = fitting_wave(pp);
    pp.wave_tokens = wave;
    if (wave == 0 && moba_workspace_size(&pp) > MOBA_NOALLOC_SCRATCH_BYTES) {
        pp.wave_tokens = 128;
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "moba_attn_fwd_noalloc: this problem needs %zu bytes of scratch even with "
                 "128-token waves; the static scratch array holds %zu bytes",
                 moba_workspace_size(&pp), (size_t)MOBA_NOALLOC_SCRATCH_BYTES);
        moba::set_error_message(msg);
        return MOBA_ERR_UNSUPPORTED;
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        moba::set_error_message(e != cudaSuccess ? cudaGetErrorString(e)
                                                 : "moba_attn_fwd_noalloc: device index too large");
        return e != cudaSuccess ? MOBA_ERR_CUDA : MOBA_ERR_UNSUPPORTED;
    }
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_setup_mutex);
        if (!g_scratch_ptr[dev]) {
            void* ptr = nullptr;
            e = cudaGetSymbolAddress(&ptr, g_scratch);
            if (e != cudaSuccess || !ptr) {
                moba::set_error_message(e != cudaSuccess ? cudaGetErrorString(e)
                                                         : "cudaGetSymbolAddress returned NULL");
                return MOBA_ERR_CUDA;
            }
            g_scratch_ptr[dev] = ptr;
        }
        scratch = g_scratch_ptr[dev];
    }
    return moba_attn_fwd(&pp, q, k, v, cu_seqlens, nullptr, nullptr, scratch,
                         MOBA_NOALLOC_SCRATCH_BYTES, out, lse, nullptr, stream);
}
