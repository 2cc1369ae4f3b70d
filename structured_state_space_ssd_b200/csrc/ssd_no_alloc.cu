// ssd_no_alloc.cu -- ssd_fwd for callers that have no way to hand it a workspace.
//
// Some callers cannot obtain device memory at the point where they run the
// layer: an inference engine that plans every buffer before serving and
// refuses allocations afterwards, a framework whose caching allocator owns
// the whole device and forbids side allocations, or a real-time loop that
// must never reach cudaMalloc (which can synchronise the device).  For them
// ssd_fwd_no_alloc uses a scratch array that the library itself places in
// device memory: a file-scope static __device__ array, created on every GPU
// that loads the library and kept until the process exits.
//
// Nothing here allocates: the array is part of the library's device image.
// Host code cannot use the array's name as a device address (on the host it
// names a host-side stand-in), so the first call on each device looks the
// address up with cudaGetSymbolAddress, with that device current, and caches
// it.  That first call may load the library's device code on the device, so
// it should come before any stream capture.
//
// Every call on a device shares the one array, and the array keeps whatever
// the last call left in it; ssd_fwd clears the status word, unit counter and
// hand-off flags it relies on at the start of each call.  Calls whose work
// overlaps on the GPU (for example on two streams) race on the array.
#include <mutex>

#include "ssd_common.cuh"

namespace {

static __device__ __align__(256) unsigned char g_no_alloc_scratch[SSD_NO_ALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch[kMaxDevices];  // device address of g_no_alloc_scratch per device, once looked up

int scratch_of_current_device(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SSD_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_no_alloc_scratch) != cudaSuccess || !p) return SSD_ERR_CUDA;
        g_scratch[dev] = p;
    }
    *out = g_scratch[dev];
    return SSD_OK;
}

}  // namespace

extern "C" int ssd_fwd_no_alloc(const void *x, const float *dt, const float *A, const void *B, const void *C,
                                const float *D, int Q, const float *init_state, void *y, float *final_state,
                                int batch, int T, int H, int P, int G, int N, int dtype, void *stream) {
    const size_t need = ssd_fwd_workspace_bytes(batch, T, H, P, G, N, Q, dtype);
    if (need == 0)  // invalid or unsupported dimensions: let ssd_fwd name the error (it launches nothing)
        return ssd_fwd(x, dt, A, B, C, D, Q, init_state, y, final_state, batch, T, H, P, G, N, dtype, nullptr, 0,
                       stream);
    if (need > (size_t)SSD_NO_ALLOC_SCRATCH_BYTES) return SSD_ERR_UNSUPPORTED;
    void *ws = nullptr;
    const int rc = scratch_of_current_device(&ws);
    if (rc != SSD_OK) return rc;
    return ssd_fwd(x, dt, A, B, C, D, Q, init_state, y, final_state, batch, T, H, P, G, N, dtype, ws,
                   (size_t)SSD_NO_ALLOC_SCRATCH_BYTES, stream);
}

extern "C" int ssd_fwd_no_alloc_check(void *stream) {
    void *ws = nullptr;
    const int rc = scratch_of_current_device(&ws);
    if (rc != SSD_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return SSD_ERR_CUDA;
    int status = 0;
    if (cudaMemcpy(&status, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SSD_ERR_CUDA;
    return status;
}
