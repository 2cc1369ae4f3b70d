// ssd_api.cu -- the extern "C" boundary of libssd.so (declared in include/ssd.h):
// argument validation, choice of launch sequence, workspace carving and the
// launches on the caller's stream.
#include <stdint.h>

#include "ssd_common.cuh"

namespace ssd {
cudaError_t launch_chunk_cumsum(const float *dt, const float *A, float *s, const Shape &sh, cudaStream_t st);
template <typename T>
cudaError_t launch_chunk_state(const T *x, const T *B, const float *s, float *S, const Shape &sh, cudaStream_t st,
                               bool from_start);
cudaError_t launch_state_passing(float *S, const float *s, const float *init, float *fin, const Shape &sh,
                                 cudaStream_t st);
template <typename T>
cudaError_t launch_chunk_scan(const T *x, const T *B, const T *C, const float *D, const float *s,
                              const float *Sprev, T *y, const Shape &sh, cudaStream_t st);
bool fused_supported(const Shape &sh, int dtype);
cudaError_t prepare_ssd_fused(const __nv_bfloat16 *x, const float *dt, const float *A, const __nv_bfloat16 *B,
                              const __nv_bfloat16 *C, const float *D, const float *init, float *fin, char *pw,
                              const Workspace &w, int *status, __nv_bfloat16 *y, const Shape &full, int p_half,
                              int n_half, const FusedDebug *dbg, const FusedGate *gate, int slot);
cudaError_t enqueue_fused_clear(char *ws, size_t stride, size_t bytes, int passes, cudaStream_t st);
cudaError_t enqueue_ssd_fused(int slot, bool after_clear, cudaStream_t st);
}  // namespace ssd

using ssd::Shape;

namespace ssd {

// Validates the dimensions of a forward or backward call; fills `sh` on success.
int check_dims(int batch, int T, int H, int P, int G, int N, int Q, int dtype, Shape *sh) {
    if (batch < 1 || T < 0 || H < 1 || P < 1 || G < 1 || N < 1 || Q < 1) return SSD_ERR_INVALID_ARG;
    if (H % G != 0) return SSD_ERR_INVALID_ARG;
    if (dtype != SSD_F32 && dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
    const int64_t bt = int64_t(batch) * T;
    if (bt * H * P > kMaxElems || bt * G * N > kMaxElems || int64_t(batch) * H * P * N > kMaxElems)
        return SSD_ERR_INVALID_ARG;
    if (P > kMaxP || N > kMaxN || Q > kMaxQ) return SSD_ERR_UNSUPPORTED;
    sh->batch = batch;
    sh->T = T;
    sh->H = H;
    sh->P = P;
    sh->G = G;
    sh->N = N;
    sh->Q = Q;
    sh->nc = (T + Q - 1) / Q;
    sh->heads_per_group = H / G;
    return SSD_OK;
}

}  // namespace ssd

namespace {

constexpr int kVersion = 200;  // 0.2.0
constexpr int kMaxStages = 8;
using ssd::check_dims;

ssd::Path choose_path(const Shape &sh, int dtype) {
    return ssd::fused_supported(sh, dtype) ? ssd::kPathFused : ssd::kPathSimt;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

const char *const kSimtStages[] = {"ssd_chunk_cumsum", "ssd_chunk_state", "ssd_state_passing", "ssd_chunk_scan"};
const char *const kFusedStages[] = {"ssd_fused"};
// launch names when the fused path splits the problem: by head columns (P = 128), state columns (N = 256)
const char *const kFusedStagesP[] = {"ssd_fused_p0_63", "ssd_fused_p64_127"};
const char *const kFusedStagesN[] = {"ssd_fused_n0_127", "ssd_fused_n128_255"};
const char *const kFusedStagesPN[] = {"ssd_fused_p0_63_n0_127", "ssd_fused_p64_127_n0_127",
                                      "ssd_fused_p0_63_n128_255", "ssd_fused_p64_127_n128_255"};

int launch_count(const Shape &sh, ssd::Path path) {
    if (sh.T == 0) return 0;
    return path == ssd::kPathFused ? ssd::fused_passes(sh) : 4;
}

// Optional event marks: ev[0] at the start of the call (before the workspace
// clear), ev[1] before the first kernel, ev[k+2] after kernel k.  A path whose
// first kernel directly follows the start (the clear being part of its first
// stage) records ev[0] alone and sets `stage0_at_start`.
struct Marks {
    cudaEvent_t *ev = nullptr;
    int n = 0;
    mutable bool stage0_at_start = false;
    bool mark(int i, cudaStream_t st) const { return !(ev && i < n) || cudaEventRecord(ev[i], st) == cudaSuccess; }
};

template <typename T>
int run_simt(const Shape &sh, const T *x, const float *dt, const float *A, const T *B, const T *C, const float *D,
             const float *init, T *y, float *fin, char *ws, const ssd::Workspace &w, cudaStream_t st,
             const Marks &mk) {
    float *s = reinterpret_cast<float *>(ws + w.s_off);
    float *S = reinterpret_cast<float *>(ws + w.state_off);
    if (!mk.mark(1, st)) return SSD_ERR_CUDA;
    if (ssd::launch_chunk_cumsum(dt, A, s, sh, st) != cudaSuccess || !mk.mark(2, st)) return SSD_ERR_CUDA;
    if (ssd::launch_chunk_state<T>(x, B, s, S, sh, st, false) != cudaSuccess || !mk.mark(3, st))
        return SSD_ERR_CUDA;
    if (ssd::launch_state_passing(S, s, init, fin, sh, st) != cudaSuccess || !mk.mark(4, st)) return SSD_ERR_CUDA;
    if (ssd::launch_chunk_scan<T>(x, B, C, D, s, S, y, sh, st) != cudaSuccess || !mk.mark(5, st))
        return SSD_ERR_CUDA;
    return SSD_OK;
}

// The fused path: every launch is worked out on the host first; then the call's marks, the clear of each
// launch's counter and flags (a kernel the first launch may overlap: it waits for the clear before any
// global access), and the launches go to the stream back to back.  The first stage's span covers the
// clear and the first launch.
int run_fused(const Shape &sh, const __nv_bfloat16 *x, const float *dt, const float *A, const __nv_bfloat16 *B,
              const __nv_bfloat16 *C, const float *D, const float *init, __nv_bfloat16 *y, float *fin, char *ws,
              const ssd::Workspace &w, cudaStream_t st, const Marks &mk, const ssd::FusedDebug *dbg,
              const ssd::FusedGate *gate) {
    // launch k covers head-column half k % pp and state-column half k / pp: the second state half adds to
    // the y its first half wrote, so it comes after both head-column launches of that first half
    const int passes = ssd::fused_passes(sh), pp = ssd::fused_p_passes(sh);
    if (passes > ssd::kMaxFusedPasses) return SSD_ERR_UNSUPPORTED;
    const size_t stride = w.total / passes;  // one launch's counter, flags and ring
    for (int k = 0; k < passes; ++k)
        if (ssd::prepare_ssd_fused(x, dt, A, B, C, D, init, fin, ws + k * stride, w,
                                   reinterpret_cast<int *>(ws + w.status_off), y, sh, k % pp, k / pp, dbg, gate,
                                   k) != cudaSuccess)
            return SSD_ERR_CUDA;
    if (!mk.mark(0, st)) return SSD_ERR_CUDA;
    mk.stage0_at_start = true;
    if (ssd::enqueue_fused_clear(ws, stride, w.clear_bytes, passes, st) != cudaSuccess) return SSD_ERR_CUDA;
    for (int k = 0; k < passes; ++k)
        if (ssd::enqueue_ssd_fused(k, k == 0, st) != cudaSuccess || !mk.mark(2 + k, st)) return SSD_ERR_CUDA;
    return SSD_OK;
}

int fwd_impl(const void *x, const float *dt, const float *A, const void *B, const void *C, const float *D, int Q,
             const float *init_state, void *y, float *final_state, int batch, int T, int H, int P, int G, int N,
             int dtype, void *workspace, size_t workspace_bytes, void *stream, const Marks &mk,
             const ssd::FusedDebug *dbg = nullptr, const ssd::FusedGate *gate = nullptr) {
    Shape sh;
    int rc = check_dims(batch, T, H, P, G, N, Q, dtype, &sh);
    if (rc != SSD_OK) return rc;
    // Per-token tensors are empty when T == 0 and may then be NULL.
    if ((T > 0 && (!x || !dt || !B || !C || !y)) || !A || !D || !workspace) return SSD_ERR_INVALID_ARG;
    const ssd::Path path = choose_path(sh, dtype);
    const size_t es = (dtype == SSD_BF16) ? 2 : 4;
    const size_t ea = (path == ssd::kPathFused) ? 16 : es;  // TMA tiles need 16-byte aligned bases
    if (!aligned(x, ea) || !aligned(B, ea) || !aligned(C, ea) || !aligned(y, ea) || !aligned(dt, 4) ||
        !aligned(A, 4) || !aligned(D, 4) || !aligned(workspace, 256) || (init_state && !aligned(init_state, 16)) ||
        (final_state && !aligned(final_state, 16)))
        return SSD_ERR_INVALID_ARG;
    const ssd::Workspace w = ssd::workspace_layout(sh, path);
    if (workspace_bytes < w.total) return SSD_ERR_INVALID_ARG;
    const size_t ybytes = es * (size_t)batch * T * H * P;
    const size_t bcbytes = es * (size_t)batch * T * G * N;
    if (ybytes && (overlaps(y, ybytes, x, ybytes) || overlaps(y, ybytes, B, bcbytes) ||
                   overlaps(y, ybytes, C, bcbytes)))
        return SSD_ERR_INVALID_ARG;
    // the gate in the fused kernel's drain: one launch with whole 64-column heads
    const bool gate_fused = gate && path == ssd::kPathFused && ssd::fused_passes(sh) == 1 && P == 64;
    if (gate) {
        if ((T > 0 && !gate->z) || !(gate->eps >= 0.f) || !aligned(gate->z, gate_fused ? 16 : es) ||
            !aligned(gate->weight, 16) || !aligned(gate->bias, 16) || (ybytes && overlaps(y, ybytes, gate->z, ybytes)))
            return SSD_ERR_INVALID_ARG;
        if (P > 4096) return SSD_ERR_UNSUPPORTED;
    }

    if (dbg && path != ssd::kPathFused) return SSD_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    if (path == ssd::kPathFused && T > 0) {
        rc = run_fused(sh, static_cast<const __nv_bfloat16 *>(x), dt, A, static_cast<const __nv_bfloat16 *>(B),
                       static_cast<const __nv_bfloat16 *>(C), D, init_state, static_cast<__nv_bfloat16 *>(y),
                       final_state, ws, w, st, mk, dbg, gate_fused ? gate : nullptr);
        // elsewhere the gate runs as its own kernel over the y just written (in place)
        if (rc == SSD_OK && gate && !gate_fused)
            rc = ssd_gate_norm(y, gate->z, gate->weight, gate->bias, y, (long long)batch * T, H * P, H, gate->eps,
                               dtype, stream);
        return rc;
    }
    if (!mk.mark(0, st)) return SSD_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, w.clear_bytes, st) != cudaSuccess) return SSD_ERR_CUDA;
    if (path == ssd::kPathFused)
        for (int k = 1; k < ssd::fused_passes(sh); ++k)
            if (cudaMemsetAsync(ws + k * (w.total / ssd::fused_passes(sh)), 0, w.clear_bytes, st) != cudaSuccess)
                return SSD_ERR_CUDA;
    if (T == 0) {
        if (!mk.mark(1, st)) return SSD_ERR_CUDA;
        if (!final_state) return SSD_OK;
        const size_t fb = sizeof(float) * (size_t)batch * H * P * N;
        cudaError_t e = init_state ? cudaMemcpyAsync(final_state, init_state, fb, cudaMemcpyDeviceToDevice, st)
                                   : cudaMemsetAsync(final_state, 0, fb, st);
        return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
    }
    if (dtype == SSD_BF16)
        rc = run_simt<__nv_bfloat16>(sh, static_cast<const __nv_bfloat16 *>(x), dt, A,
                                     static_cast<const __nv_bfloat16 *>(B), static_cast<const __nv_bfloat16 *>(C), D,
                                     init_state, static_cast<__nv_bfloat16 *>(y), final_state, ws, w, st, mk);
    else
        rc = run_simt<float>(sh, static_cast<const float *>(x), dt, A, static_cast<const float *>(B),
                             static_cast<const float *>(C), D, init_state, static_cast<float *>(y), final_state, ws,
                             w, st, mk);
    // elsewhere the gate runs as its own kernel over the y just written (in place)
    if (rc == SSD_OK && gate && !gate_fused)
        rc = ssd_gate_norm(y, gate->z, gate->weight, gate->bias, y, (long long)batch * T, H * P, H, gate->eps, dtype,
                           stream);
    return rc;
}

}  // namespace

extern "C" {

size_t ssd_fwd_workspace_bytes(int batch, int T, int H, int P, int G, int N, int Q, int dtype) {
    Shape sh;
    if (check_dims(batch, T, H, P, G, N, Q, dtype, &sh) != SSD_OK) return 0;
    return ssd::workspace_layout(sh, choose_path(sh, dtype)).total;
}

int ssd_fwd_launch_count(int batch, int T, int H, int P, int G, int N, int Q, int dtype) {
    Shape sh;
    if (check_dims(batch, T, H, P, G, N, Q, dtype, &sh) != SSD_OK) return 0;
    return launch_count(sh, choose_path(sh, dtype));
}

const char *ssd_fwd_stage_name(int batch, int T, int H, int P, int G, int N, int Q, int dtype, int i) {
    Shape sh;
    if (check_dims(batch, T, H, P, G, N, Q, dtype, &sh) != SSD_OK) return nullptr;
    const ssd::Path path = choose_path(sh, dtype);
    if (i < 0 || i >= launch_count(sh, path)) return nullptr;
    if (path != ssd::kPathFused) return kSimtStages[i];
    const int pp = ssd::fused_p_passes(sh), np = ssd::fused_n_passes(sh);
    if (pp == 2 && np == 2) return kFusedStagesPN[i];
    if (pp == 2) return kFusedStagesP[i];
    if (np == 2) return kFusedStagesN[i];
    return kFusedStages[i];
}

int ssd_fwd(const void *x, const float *dt, const float *A, const void *B, const void *C, const float *D, int Q,
            const float *init_state, void *y, float *final_state, int batch, int T, int H, int P, int G, int N,
            int dtype, void *workspace, size_t workspace_bytes, void *stream) {
    return fwd_impl(x, dt, A, B, C, D, Q, init_state, y, final_state, batch, T, H, P, G, N, dtype, workspace,
                    workspace_bytes, stream, Marks{});
}

int ssd_fwd_timed(const void *x, const float *dt, const float *A, const void *B, const void *C, const float *D,
                  int Q, const float *init_state, void *y, float *final_state, int batch, int T, int H, int P,
                  int G, int N, int dtype, void *workspace, size_t workspace_bytes, void *stream, float *stage_ms,
                  int max_stages, float *total_ms) {
    // One set of events per device, created on that device the first time this
    // host thread times a call there, kept until the process exits.
    constexpr int kMaxDevices = 64;
    thread_local cudaEvent_t events[kMaxDevices][kMaxStages + 2];
    thread_local bool created[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SSD_ERR_CUDA;
    if (!created[dev]) {
        for (int i = 0; i < kMaxStages + 2; ++i)
            if (cudaEventCreate(&events[dev][i]) != cudaSuccess) return SSD_ERR_CUDA;
        created[dev] = true;
    }
    Shape sh;
    int rc = check_dims(batch, T, H, P, G, N, Q, dtype, &sh);
    if (rc != SSD_OK) return rc;
    const int k = launch_count(sh, choose_path(sh, dtype));
    Marks mk;
    mk.ev = events[dev];
    mk.n = k + 2;
    rc = fwd_impl(x, dt, A, B, C, D, Q, init_state, y, final_state, batch, T, H, P, G, N, dtype, workspace,
                  workspace_bytes, stream, mk);
    if (rc != SSD_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return SSD_ERR_CUDA;
    for (int i = 0; i < k && i < max_stages && stage_ms; ++i)
        if (cudaEventElapsedTime(&stage_ms[i], events[dev][(i == 0 && mk.stage0_at_start) ? 0 : i + 1],
                                 events[dev][i + 2]) != cudaSuccess)
            return SSD_ERR_CUDA;
    if (total_ms) {
        *total_ms = 0.f;
        if (k > 0 && cudaEventElapsedTime(total_ms, events[dev][0], events[dev][k + 1]) != cudaSuccess)
            return SSD_ERR_CUDA;
    }
    return SSD_OK;
}

int ssd_fwd_gated(const void *x, const float *dt, const float *A, const void *B, const void *C, const float *D,
                  int Q, const float *init_state, const void *z, const float *norm_weight, const float *norm_bias,
                  float eps, void *out, float *final_state, int batch, int T, int H, int P, int G, int N, int dtype,
                  void *workspace, size_t workspace_bytes, void *stream) {
    ssd::FusedGate gate{z, norm_weight, norm_bias, eps};
    return fwd_impl(x, dt, A, B, C, D, Q, init_state, out, final_state, batch, T, H, P, G, N, dtype, workspace,
                    workspace_bytes, stream, Marks{}, nullptr, &gate);
}

int ssd_fwd_gated_launch_count(int batch, int T, int H, int P, int G, int N, int Q, int dtype) {
    Shape sh;
    if (check_dims(batch, T, H, P, G, N, Q, dtype, &sh) != SSD_OK) return 0;
    const ssd::Path path = choose_path(sh, dtype);
    const int k = launch_count(sh, path);
    if (k == 0) return 0;
    return (path == ssd::kPathFused && ssd::fused_passes(sh) == 1 && P == 64) ? k : k + 1;
}

int ssd_fwd_withhold_publish(const void *x, const float *dt, const float *A, const void *B, const void *C,
                             const float *D, int Q, const float *init_state, void *y, float *final_state, int batch,
                             int T, int H, int P, int G, int N, int dtype, void *workspace, size_t workspace_bytes,
                             void *stream, int withhold_b, int withhold_h, int withhold_c, unsigned flag_polls) {
    if (withhold_b < 0 || withhold_b >= batch || withhold_h < 0 || withhold_h >= H || withhold_c < 0 ||
        flag_polls == 0)
        return SSD_ERR_INVALID_ARG;
    ssd::FusedDebug dbg;
    dbg.flag_polls = flag_polls;
    dbg.withhold_bh = withhold_b * H + withhold_h;
    dbg.withhold_c = withhold_c;
    return fwd_impl(x, dt, A, B, C, D, Q, init_state, y, final_state, batch, T, H, P, G, N, dtype, workspace,
                    workspace_bytes, stream, Marks{}, &dbg);
}

int ssd_fwd_check(const void *workspace, void *stream) {
    if (!workspace) return SSD_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return SSD_ERR_CUDA;
    int status = 0;
    if (cudaMemcpy(&status, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SSD_ERR_CUDA;
    return status;
}

const char *ssd_status_string(int status) {
    switch (status) {
        case SSD_OK: return "ok";
        case SSD_ERR_INVALID_ARG: return "invalid argument";
        case SSD_ERR_UNSUPPORTED: return "unsupported shape (P <= 128, N <= 256, Q <= 256)";
        case SSD_ERR_CUDA: return "CUDA error";
        case SSD_ERR_TIMEOUT: return "a bounded device-side wait timed out";
        default: return "unknown status";
    }
}

int ssd_version(void) { return kVersion; }

}  // extern "C"
