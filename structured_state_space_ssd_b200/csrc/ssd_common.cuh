// ssd_common.cuh -- small shared helpers of the libssd.so kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/ssd.h"

namespace ssd {

// Element load/store for the two input dtypes; arithmetic is always fp32.
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// 16 bytes of T as fp32: four floats or eight bf16 (a bf16 is the top half of its fp32).
__device__ __forceinline__ void unpack16(const uint4 &u, float *f, float) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ void unpack16(const uint4 &u, float *f, __nv_bfloat16) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// dst[r * dld + k] = src[r * ld + k] as fp32 for r < rows and k < cols, zero for rows r >= valid and
// for columns k in [cols, cols_pad).  With vec (src and ld 16-byte aligned, cols a multiple of the
// vector) each thread issues up to four 16-byte loads before it stores any.  All 256 threads call it.
template <typename T>
__device__ __forceinline__ void stage_rows(float *dst, int dld, const T *src, size_t ld, int rows, int valid,
                                           int cols, int cols_pad, bool vec) {
    if (vec) {
        constexpr int VE = 16 / (int)sizeof(T);
        const int cpr = cols / VE, total = rows * cpr;
        for (int base = threadIdx.x; base < total; base += 4 * 256) {
            uint4 u[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int idx = base + q * 256;
                const int r = idx / cpr, kc = idx - r * cpr;
                u[q] = make_uint4(0u, 0u, 0u, 0u);
                if (idx < total && r < valid)
                    u[q] = __ldg(reinterpret_cast<const uint4 *>(src + (size_t)r * ld + (size_t)kc * VE));
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int idx = base + q * 256;
                if (idx < total) {
                    const int r = idx / cpr, kc = idx - r * cpr;
                    float f[VE];
                    unpack16(u[q], f, T());
                    float4 *d = reinterpret_cast<float4 *>(dst + r * dld + kc * VE);
#pragma unroll
                    for (int e = 0; e < VE / 4; ++e)
                        d[e] = make_float4(f[4 * e], f[4 * e + 1], f[4 * e + 2], f[4 * e + 3]);
                }
            }
        }
    } else {
        for (int idx = threadIdx.x; idx < rows * cols; idx += 256) {
            const int r = idx / cols, k = idx - r * cols;
            dst[r * dld + k] = r < valid ? to_f32(src[(size_t)r * ld + k]) : 0.f;
        }
    }
    const int padc = cols_pad - cols;
    for (int idx = threadIdx.x; idx < rows * padc; idx += 256) {
        const int r = idx / padc, k = cols + (idx - r * padc);
        dst[r * dld + k] = 0.f;
    }
}

// Problem shape as every kernel sees it.
struct Shape {
    int batch, T, H, P, G, N, Q, nc;
    int heads_per_group;  // H / G
};

// The fused path's inter-chunk chain.  The owner of chunk c forms the outgoing state
// S~_c = exp(sigma_c) S~_{c-1} + L_c from the one before.  With look-back depth D > 1 every owner
// also publishes its local state L_c and total decay sigma_c as soon as its products are done, and
// the owner of chunk c starts from the most recent published S~_j with j >= c - D, folding in
// L_{j+1} .. L_{c-1} (the decoupled look-back of a single-pass scan), so that a long sequence is not
// bound by one hand-off per chunk.  This is valid because the chunk recurrence is a 1-semiseparable
// product, associative on (decay, state) pairs ("Transformers are SSMs", analysis page, section "The
// 1-Semiseparable Matrix: Building Block for Everything": the associative-scan decomposition).  D > 1 is used where the chain would be long and the ring, twice
// as large, stays small enough to live in L2.  `s` is one launch's shape (64 head columns, at most
// 128 state columns).
inline int fused_lookback(const Shape &s) {
    const size_t bh = (size_t)s.batch * s.H;
    const size_t slot_bytes = 2 * sizeof(float) * 64 * (size_t)s.N;  // S~ and L
    return (s.nc >= 32 && bh * 8 * slot_bytes <= (size_t(48) << 20)) ? 4 : 1;
}
// Ring slots per (batch, head): chunk c's states go to slot c % R.  Three with D = 1; 2D with look-back,
// so that the slot an owner overwrites was last read by owners at least D chunks back.  With D = 1 only
// the bf16 state tiles (read by the other blocks) use the R slots: the fp32 state is read by the next
// owner alone, which reads S~_{c-1} and writes S~_c in place, so it has one slot.  (With look-back
// the other blocks read S~ from the fp32 slots, which the owners read too: there are no tiles.)
inline int fused_ring_slots(int d) { return d == 1 ? 3 : 2 * d; }
// fp32 floats per (batch, head): one slot of S~ (64 x N) with D = 1; R slots of S~ and L with look-back
inline size_t fused_ring_floats(const Shape &s, int d) {
    return d == 1 ? (size_t)64 * s.N : (size_t)fused_ring_slots(d) * 2 * 64 * s.N;
}
// Rows of a bf16 state tile: the K extent of the inter-chunk product (N rounded up to 64; rows past N zero).
inline int fused_tile_rows(const Shape &s) { return (s.N + 63) / 64 * 64; }

// The two launch sequences: stage-per-kernel on CUDA cores (any shape and
// dtype within the limits) or the fused tensor-core kernel (bf16, P a multiple
// of 8 up to 64 or P = 128, N a multiple of 16 up to 128 or N = 256, Q in
// {128, 256}).
enum Path { kPathSimt = 0, kPathFused = 1 };

// Gate and per-head GroupNorm applied in the fused kernel's drain (ssd_fwd_gated): z as x, bf16;
// weight and bias [H * P] fp32 or null.
struct FusedGate {
    const void *z;
    const float *weight, *bias;
    float eps;
};

// Test hooks of the fused kernel's hand-off (ssd_fwd_withhold_publish):
// each wait on another CTA's flag gives up after flag_polls polls (0: the
// default bound), and the owner of chunk withhold_c of sequence withhold_bh
// (batch * H + head) never publishes its state (-1: every owner publishes).
struct FusedDebug {
    unsigned flag_polls;
    int withhold_bh;
    int withhold_c;
};

// Workspace carve-up, computed identically by ssd_fwd_workspace_bytes and ssd_fwd.
// The front 256-byte block holds the status word and the unit counter; it and
// the per-(batch, head) flags after it are cleared at the start of every call
// (on the fused path by a small kernel the first launch depends on, elsewhere
// by a memset).
struct Workspace {
    size_t status_off;  // int status word
    size_t counter_off; // int unit counter (fused path)
    size_t inc_off;     // fused path: int inc[batch * H][R] (one count per sequence without look-back)
    size_t tin_off;     // fused path, D = 1: int tin[batch * H][R], c + 1 once the bf16 tile of S~_c is in slot c % R
    size_t agg_off;     // fused path: int agg[batch * H][R], c + 1 once L_c and sigma_c are in slot c % R
    size_t cons_off;    // fused path: int cons[batch * H][R], reads of the slot so far (a count)
    size_t sig_off;     // fused path: float sigma[batch * H][R], chunk c's total log2 decay in slot c % R
    size_t clear_bytes; // bytes from offset 0 cleared per call
    size_t s_off;       // CUDA-core path: float s[batch][H][nc][Q], inclusive log-decay prefix sums per chunk
    size_t state_off;   // CUDA-core path: float S[batch][nc][H][P][N], chunk states then entering states
    size_t ring_off;    // fused path: float ring[batch][H][1, or R x 2][16][N][4], states of recent chunks
    size_t tile_off;    // fused path, D = 1: bf16 tile[batch * H][R][rows][64], S~ in the MMA's 128-byte swizzle
    size_t total;
};

// Dimension limits shared by the forward and backward entry points.
constexpr int kMaxP = 128, kMaxN = 256, kMaxQ = 256;
constexpr int64_t kMaxElems = int64_t(1) << 46;

// Validates the dimensions of a forward or backward call; fills `sh` on success
// (ssd_api.cu).
int check_dims(int batch, int T, int H, int P, int G, int N, int Q, int dtype, Shape *sh);

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// The backward's head-summing scans (bf16, Q a multiple of 128) keep, for dB and for dC, one partial sum
// of 128 rows per (CTA, (chunk, 128-row block, group)) pair, in slot CTA + pair (at most kBwdSumMaxCtas
// CTAs), and two half-row dot products per (batch, token, head).
constexpr int kBwdSumMaxCtas = 256;
inline size_t bwd_sum_bytes(const Shape &s) {
    if (s.Q % 128 != 0) return 0;
    const size_t keys = (size_t)s.batch * s.nc * (s.Q / 128) * s.G;
    return align256(sizeof(float) * (kBwdSumMaxCtas + keys) * 128 * s.N) +
           align256(sizeof(float) * 2 * (size_t)s.batch * s.T * s.H);
}
inline size_t bwd_sum_dot_off(const Shape &s) {
    const size_t keys = (size_t)s.batch * s.nc * (s.Q / 128) * s.G;
    return align256(sizeof(float) * (kBwdSumMaxCtas + keys) * 128 * s.N);
}

// The fused path works on 64 head columns and up to 128 state columns per launch: P = 128 runs as two
// launches over column halves of x and y, N = 256 as two over halves of the state (the second adding to
// y).  Each launch has its own counter, flags and ring (one after the other in the workspace); the
// status word is shared.  A head dimension below 64 is zero-padded, so the ring always has 64 rows.
inline int fused_p_passes(const Shape &s) { return s.P > 64 ? 2 : 1; }
inline int fused_n_passes(const Shape &s) { return s.N > 128 ? 2 : 1; }
inline int fused_passes(const Shape &s) { return fused_p_passes(s) * fused_n_passes(s); }
constexpr int kMaxFusedPasses = 4;

inline Workspace workspace_layout_one(const Shape &s, Path path);

inline Workspace workspace_layout(const Shape &s, Path path) {
    if (path != kPathFused) return workspace_layout_one(s, path);
    Shape h = s;
    h.P = 64;
    if (h.N > 128) h.N = 128;
    Workspace w = workspace_layout_one(h, path);
    w.total *= fused_passes(s);  // launch k's counter, flags and ring sit at k * (total / passes)
    return w;
}

inline Workspace workspace_layout_one(const Shape &s, Path path) {
    Workspace w;
    const size_t bh = (size_t)s.batch * s.H;
    w.status_off = 0;
    w.counter_off = 4;
    size_t off = 256;
    const int d = (path == kPathFused) ? fused_lookback(s) : 1, R = fused_ring_slots(d);
    const size_t per_slot = (d == 1) ? 0 : bh * R;  // agg and sigma: look-back only
    w.inc_off = off;
    off += sizeof(int) * (d == 1 ? bh : bh * R);
    w.tin_off = off;
    off += sizeof(int) * (d == 1 ? bh * R : 0);
    w.cons_off = off;
    off += sizeof(int) * bh * R;
    w.agg_off = off;
    off += sizeof(int) * per_slot;
    w.sig_off = off;
    off += sizeof(float) * per_slot;
    off = align256(off);
    w.clear_bytes = (path == kPathFused) ? off : 256;
    w.s_off = off;
    if (path != kPathFused) off = align256(off + sizeof(float) * bh * s.nc * s.Q);
    w.state_off = w.ring_off = off;
    w.tile_off = off;
    if (path == kPathFused) {
        off = align256(off + sizeof(float) * bh * fused_ring_floats(s, d));
        w.tile_off = off;
        if (d == 1) off = align256(off + sizeof(uint16_t) * bh * R * fused_tile_rows(s) * 64);
    } else
        off = align256(off + sizeof(float) * (size_t)s.batch * s.nc * s.H * s.P * s.N);
    w.total = off;
    return w;
}

}  // namespace ssd
