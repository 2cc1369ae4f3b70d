// ssd_step.cu -- one autoregressive step of the SSD recurrence (decode).
//
// The recurrent mode of the layer ("Transformers are SSMs", analysis page,
// section "The Scalar-Identity SSM"; the English note's section "Working
// Through Four Tokens" advances it by hand one token at a time): for every
// batch row b and head h, with g = h / (H / G),
//
//     state[b,h] = exp(dt[b,h] * A[h]) * state[b,h] + x[b,h] B[b,g]^T     (P x N, in place)
//     y[b,h]     = state[b,h] C[b,g] + D[h] * x[b,h]
//
// The work is one read and one write of the fp32 state per token, so the
// step is bound by memory bandwidth (HBM, or L2 when a decode loop keeps the
// state resident).  Layout: one warp per 4 state rows of one (b, h); its lanes
// walk the rows' N values four at a time (16-byte loads and stores, all four
// rows' loads issued before any use, B and C read once for the four) when N
// is a multiple of 4 and the state is 16-byte aligned, one at a time
// otherwise, and warp reductions form y[b,h,p].  32 rows per 256-thread block.
#include "ssd_common.cuh"

namespace ssd {

namespace {

constexpr int kStepWarps = 8;
constexpr int kRowsPerWarp = 4;  // state rows per warp: 4 x 16 bytes in flight per lane

template <typename T>
__device__ __forceinline__ void load4(const T *p, float (&v)[4]);

template <>
__device__ __forceinline__ void load4<float>(const float *p, float (&v)[4]) {
    const float4 q = *reinterpret_cast<const float4 *>(p);
    v[0] = q.x;
    v[1] = q.y;
    v[2] = q.z;
    v[3] = q.w;
}

template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[4]) {
    const uint2 q = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&q.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&q.y);
    v[0] = __low2float(lo);
    v[1] = __high2float(lo);
    v[2] = __low2float(hi);
    v[3] = __high2float(hi);
}

template <typename T, bool kVec>
__global__ void __launch_bounds__(kStepWarps * 32)
    ssd_step_kernel(float *__restrict__ state, const T *__restrict__ x, const float *__restrict__ dt,
                    const float *__restrict__ A, const T *__restrict__ B, const T *__restrict__ C,
                    const float *__restrict__ D, T *__restrict__ y, int H, int P, int G, int N) {
    const int lane = threadIdx.x & 31;
    const int p0 = (blockIdx.x * kStepWarps + (threadIdx.x >> 5)) * kRowsPerWarp;
    const int h = blockIdx.y, b = blockIdx.z;
    if (p0 >= P) return;
    const int g = h / (H / G);
    const size_t bh = (size_t)b * H + h;
    const float a = expf(dt[bh] * A[h]);
    float xv[kRowsPerWarp], acc[kRowsPerWarp];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        xv[r] = p0 + r < P ? to_f32(x[bh * P + p0 + r]) : 0.f;
        acc[r] = 0.f;
    }
    float *rows = state + (bh * P + p0) * N;
    const T *Bg = B + ((size_t)b * G + g) * N;
    const T *Cg = C + ((size_t)b * G + g) * N;
    if (kVec) {
        for (int n = lane * 4; n < N; n += 128) {
            // every row's values first (more loads in flight), then B and C once for all rows
            float4 s[kRowsPerWarp];
#pragma unroll
            for (int r = 0; r < kRowsPerWarp; ++r)
                if (p0 + r < P) s[r] = *reinterpret_cast<const float4 *>(rows + (size_t)r * N + n);
            float bv[4], cv[4];
            load4<T>(Bg + n, bv);
            load4<T>(Cg + n, cv);
#pragma unroll
            for (int r = 0; r < kRowsPerWarp; ++r) {
                if (p0 + r >= P) continue;
                s[r].x = fmaf(a, s[r].x, xv[r] * bv[0]);
                s[r].y = fmaf(a, s[r].y, xv[r] * bv[1]);
                s[r].z = fmaf(a, s[r].z, xv[r] * bv[2]);
                s[r].w = fmaf(a, s[r].w, xv[r] * bv[3]);
                *reinterpret_cast<float4 *>(rows + (size_t)r * N + n) = s[r];
                acc[r] = fmaf(s[r].x, cv[0], acc[r]);
                acc[r] = fmaf(s[r].y, cv[1], acc[r]);
                acc[r] = fmaf(s[r].z, cv[2], acc[r]);
                acc[r] = fmaf(s[r].w, cv[3], acc[r]);
            }
        }
    } else {
        for (int n = lane; n < N; n += 32) {
            const float bn = to_f32(Bg[n]), cn = to_f32(Cg[n]);
#pragma unroll
            for (int r = 0; r < kRowsPerWarp; ++r) {
                if (p0 + r >= P) continue;
                float *e = rows + (size_t)r * N + n;
                const float v = fmaf(a, *e, xv[r] * bn);
                *e = v;
                acc[r] = fmaf(v, cn, acc[r]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], o);
        if (lane == 0 && p0 + r < P) y[bh * P + p0 + r] = from_f32<T>(acc[r] + D[h] * xv[r]);
    }
}

template <typename T>
cudaError_t launch_step(float *state, const void *x, const float *dt, const float *A, const void *B, const void *C,
                        const float *D, void *y, int batch, int H, int P, int G, int N, bool vec, cudaStream_t st) {
    const int rows_per_block = kStepWarps * kRowsPerWarp;
    const dim3 grid((P + rows_per_block - 1) / rows_per_block, H, batch);
    if (vec)
        ssd_step_kernel<T, true><<<grid, kStepWarps * 32, 0, st>>>(
            state, static_cast<const T *>(x), dt, A, static_cast<const T *>(B), static_cast<const T *>(C), D,
            static_cast<T *>(y), H, P, G, N);
    else
        ssd_step_kernel<T, false><<<grid, kStepWarps * 32, 0, st>>>(
            state, static_cast<const T *>(x), dt, A, static_cast<const T *>(B), static_cast<const T *>(C), D,
            static_cast<T *>(y), H, P, G, N);
    return cudaGetLastError();
}

bool is_aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool ranges_overlap(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t u = reinterpret_cast<uintptr_t>(a), v = reinterpret_cast<uintptr_t>(b);
    return u < v + nb && v < u + na;
}

}  // namespace

}  // namespace ssd

extern "C" int ssd_step(float *state, const void *x, const float *dt, const float *A, const void *B, const void *C,
                        const float *D, void *y, int batch, int H, int P, int G, int N, int dtype, void *stream) {
    constexpr int kMaxStepN = 1024, kMaxRows = 65535;
    if (!state || !x || !dt || !A || !B || !C || !D || !y) return SSD_ERR_INVALID_ARG;
    if (batch < 1 || H < 1 || P < 1 || G < 1 || N < 1 || H % G != 0) return SSD_ERR_INVALID_ARG;
    if (dtype != SSD_F32 && dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
    if (N > kMaxStepN || batch > kMaxRows || H > kMaxRows) return SSD_ERR_UNSUPPORTED;
    if ((int64_t)batch * H * P * N > (int64_t(1) << 40)) return SSD_ERR_INVALID_ARG;
    const size_t es = dtype == SSD_BF16 ? 2 : 4;
    if (!ssd::is_aligned(state, 4) || !ssd::is_aligned(x, es) || !ssd::is_aligned(B, es) ||
        !ssd::is_aligned(C, es) || !ssd::is_aligned(y, es) || !ssd::is_aligned(dt, 4) || !ssd::is_aligned(A, 4) ||
        !ssd::is_aligned(D, 4))
        return SSD_ERR_INVALID_ARG;
    const size_t ybytes = es * (size_t)batch * H * P;
    const size_t sbytes = 4 * (size_t)batch * H * P * N;
    const size_t bcbytes = es * (size_t)batch * G * N;
    if (ssd::ranges_overlap(y, ybytes, x, ybytes) || ssd::ranges_overlap(y, ybytes, state, sbytes) ||
        ssd::ranges_overlap(y, ybytes, B, bcbytes) || ssd::ranges_overlap(y, ybytes, C, bcbytes) ||
        ssd::ranges_overlap(state, sbytes, x, ybytes) || ssd::ranges_overlap(state, sbytes, B, bcbytes) ||
        ssd::ranges_overlap(state, sbytes, C, bcbytes))
        return SSD_ERR_INVALID_ARG;
    // 16-byte state rows, and B/C rows whose 4-element groups are 16 (fp32) or 8 (bf16) bytes aligned
    const bool vec = N % 4 == 0 && ssd::is_aligned(state, 16) && ssd::is_aligned(B, 4 * es) &&
                     ssd::is_aligned(C, 4 * es);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e =
        dtype == SSD_BF16
            ? ssd::launch_step<__nv_bfloat16>(state, x, dt, A, B, C, D, y, batch, H, P, G, N, vec, st)
            : ssd::launch_step<float>(state, x, dt, A, B, C, D, y, batch, H, P, G, N, vec, st);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
