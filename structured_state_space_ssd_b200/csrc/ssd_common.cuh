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

// Problem shape as every kernel sees it.
struct Shape {
    int batch, T, H, P, G, N, Q, nc;
    int heads_per_group;  // H / G
};

// Workspace carve-up, computed identically by ssd_fwd_workspace_bytes and ssd_fwd.
struct Workspace {
    size_t status_off;  // int status word (+ padding)
    size_t s_off;       // float s[batch][H][nc][Q]: inclusive log-decay prefix sums per chunk
    size_t state_off;   // float S[batch][nc][H][P][N]: chunk states, then the state entering each chunk
    size_t total;
};

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

inline Workspace workspace_layout(const Shape &s) {
    Workspace w;
    size_t off = 0;
    w.status_off = off;
    off = align256(off + 256);
    w.s_off = off;
    off = align256(off + sizeof(float) * (size_t)s.batch * s.H * s.nc * s.Q);
    w.state_off = off;
    off = align256(off + sizeof(float) * (size_t)s.batch * s.nc * s.H * s.P * s.N);
    w.total = off;
    return w;
}

}  // namespace ssd
