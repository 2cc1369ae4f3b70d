// ssd_gate_norm.cu -- the Mamba-2 block's step after the SSD layer: gate, then GroupNorm.
//
// "Transformers are SSMs" (analysis page, section "The Mamba-2 Architecture",
// paragraphs "Gating" and "Extra normalization"): the layer output y is gated
// by the Swish of a parallel branch z, g = y * silu(z), and GroupNorm follows.
// Per token, the C = H * P channels split into ngroups contiguous groups of
// gs = C / ngroups channels, and per group
//
//     out = (g - mean(g)) * rsqrt(var(g) + eps) * weight + bias
//
// with the population variance.  One read of y and z and one write of out:
// bound by memory bandwidth.  One warp per (token, group): the gated values go
// to a per-warp shared-memory row once, then the mean, the variance (two
// passes, no cancellation) and the output are formed from it.  Groups of 8 to
// 256 channels (a group per head, for one) take a register path instead: 8
// channels per lane, 1 to 32 lanes per group.  out may be y itself: every
// value is read before it is written, by the thread that writes it.
#include "ssd_common.cuh"

namespace ssd {

namespace {

constexpr int kGnWarps = 8;
constexpr int kGnMaxGroup = 4096;  // channels per group held in shared memory (16 KB per warp)

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// z * sigmoid(z) with the fast exponential and reciprocal: the kernel is otherwise bound by issue,
// not by memory (for very negative z the reciprocal of an infinite denominator is 0)
__device__ __forceinline__ float silu(float z) { return z * __frcp_rn(1.f + __expf(-z)); }

template <typename T>
__global__ void __launch_bounds__(kGnWarps * 32)
    gate_norm_kernel(const T *y, const T *__restrict__ z, const float *__restrict__ weight,
                     const float *__restrict__ bias, T *out, long long units, int C, int gs, float eps,
                     bool vec_ok) {
    extern __shared__ float gn_smem[];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const long long unit = (long long)blockIdx.x * kGnWarps + w;  // (token, group)
    if (unit >= units) return;
    const int ng = C / gs;
    const long long token = unit / ng;
    const int c0 = (int)(unit % ng) * gs;
    const size_t base = (size_t)token * C + c0;
    float *g = gn_smem + (size_t)w * gs;
    float sum = 0.f;
    bool vec = false;
    if constexpr (sizeof(T) == 2) vec = vec_ok && gs % 8 == 0 && (base % 8) == 0;
    if (vec) {
        // 8 bf16 values (16 bytes) per load
        for (int i = lane * 8; i < gs; i += 256) {
            const uint4 yv = *reinterpret_cast<const uint4 *>(y + base + i);
            const uint4 zv = *reinterpret_cast<const uint4 *>(z + base + i);
            const __nv_bfloat16 *ye = reinterpret_cast<const __nv_bfloat16 *>(&yv);
            const __nv_bfloat16 *ze = reinterpret_cast<const __nv_bfloat16 *>(&zv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float v = __bfloat162float(ye[e]) * silu(__bfloat162float(ze[e]));
                g[i + e] = v;
                sum += v;
            }
        }
    } else {
        for (int i = lane; i < gs; i += 32) {
            const float v = to_f32(y[base + i]) * silu(to_f32(z[base + i]));
            g[i] = v;
            sum += v;
        }
    }
    const float mean = warp_sum(sum) / gs;
    float sq = 0.f;
    for (int i = lane; i < gs; i += 32) {
        const float d = g[i] - mean;
        sq = fmaf(d, d, sq);
    }
    const float rstd = rsqrtf(warp_sum(sq) / gs + eps);
    for (int i = lane; i < gs; i += 32) {
        float v = (g[i] - mean) * rstd;
        if (weight) v *= weight[c0 + i];
        if (bias) v += bias[c0 + i];
        out[base + i] = from_f32<T>(v);
    }
}

// 8 values of one row at p (16-byte aligned) as floats, and back
template <typename T>
__device__ __forceinline__ void load8(const T *p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 q = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&q);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __bfloat162float(e[i]);
}
template <>
__device__ __forceinline__ void load8<float>(const float *p, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}
template <typename T>
__device__ __forceinline__ void store8(T *p, const float (&v)[8]);
template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16 *p, const float (&v)[8]) {
    uint4 q;
    __nv_bfloat16 *e = reinterpret_cast<__nv_bfloat16 *>(&q);
#pragma unroll
    for (int i = 0; i < 8; ++i) e[i] = __float2bfloat16_rn(v[i]);
    *reinterpret_cast<uint4 *>(p) = q;
}
template <>
__device__ __forceinline__ void store8<float>(float *p, const float (&v)[8]) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4 *>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// Groups of 8 * L channels (L = 1, 2, .., 32 lanes per group, 32 / L groups per warp): every lane
// holds 8 consecutive channels in registers, the group's sums are shuffle reductions over its L lanes.
// Groups are numbered in memory order (token-major), so a group's channels start at unit * gs and its
// channel offset within the token is (unit % ngroups) * gs (32-bit arithmetic when it fits).
template <typename T, int L>
__global__ void __launch_bounds__(kGnWarps * 32)
    gate_norm_small_kernel(const T *y, const T *__restrict__ z, const float *__restrict__ weight,
                           const float *__restrict__ bias, T *out, long long units, int ngroups, float eps) {
    constexpr int gs = 8 * L;
    const long long t = (long long)blockIdx.x * kGnWarps * 32 + threadIdx.x;
    const long long unit = t / L;
    const bool active = unit < units;
    const int sub = (int)(t & (L - 1));
    const size_t base = (size_t)(active ? unit : 0) * gs + sub * 8;
    float g[8], zv[8];
    float sum = 0.f;
    if (active) {
        load8<T>(y + base, g);
        load8<T>(z + base, zv);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            g[i] *= silu(zv[i]);
            sum += g[i];
        }
    }
#pragma unroll
    for (int o = 1; o < L; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float mean = sum * (1.f / gs);
    float sq = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float d = g[i] - mean;
        sq = fmaf(d, d, sq);
    }
#pragma unroll
    for (int o = 1; o < L; o <<= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (!active) return;
    const float rstd = rsqrtf(sq * (1.f / gs) + eps);
    if (weight || bias) {
        const int grp = units < (1LL << 31) ? (int)unit % ngroups : (int)(unit % ngroups);
        const int c = grp * gs + sub * 8;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            g[i] = fmaf((g[i] - mean) * rstd, weight ? weight[c + i] : 1.f, bias ? bias[c + i] : 0.f);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) g[i] = (g[i] - mean) * rstd;
    }
    store8<T>(out + base, g);
}

template <typename T, int L>
cudaError_t launch_small(const void *y, const void *z, const float *weight, const float *bias, void *out,
                         long long units, int ngroups, float eps, cudaStream_t st) {
    const long long threads = units * L;
    const long long blocks = (threads + kGnWarps * 32 - 1) / (kGnWarps * 32);
    gate_norm_small_kernel<T, L><<<(unsigned)blocks, kGnWarps * 32, 0, st>>>(
        static_cast<const T *>(y), static_cast<const T *>(z), weight, bias, static_cast<T *>(out), units, ngroups,
        eps);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_gate_norm(const void *y, const void *z, const float *weight, const float *bias, void *out,
                             long long rows, int C, int ngroups, float eps, bool vec_ok, cudaStream_t st) {
    const int gs = C / ngroups;
    const long long units = rows * ngroups;
    if (vec_ok) {
        switch (gs) {
            case 8: return launch_small<T, 1>(y, z, weight, bias, out, units, ngroups, eps, st);
            case 16: return launch_small<T, 2>(y, z, weight, bias, out, units, ngroups, eps, st);
            case 32: return launch_small<T, 4>(y, z, weight, bias, out, units, ngroups, eps, st);
            case 64: return launch_small<T, 8>(y, z, weight, bias, out, units, ngroups, eps, st);
            case 128: return launch_small<T, 16>(y, z, weight, bias, out, units, ngroups, eps, st);
            case 256: return launch_small<T, 32>(y, z, weight, bias, out, units, ngroups, eps, st);
            default: break;
        }
    }
    const long long blocks = (units + kGnWarps - 1) / kGnWarps;
    const size_t smem = (size_t)kGnWarps * gs * sizeof(float);
    if (smem > 48 * 1024) {
        const cudaError_t e =
            cudaFuncSetAttribute(gate_norm_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    gate_norm_kernel<T><<<(unsigned)blocks, kGnWarps * 32, smem, st>>>(
        static_cast<const T *>(y), static_cast<const T *>(z), weight, bias, static_cast<T *>(out), units, C, gs,
        eps, vec_ok);
    return cudaGetLastError();
}

bool gn_aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool gn_overlap(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t u = reinterpret_cast<uintptr_t>(a), v = reinterpret_cast<uintptr_t>(b);
    return u < v + nb && v < u + na;
}

}  // namespace

}  // namespace ssd

extern "C" int ssd_gate_norm(const void *y, const void *z, const float *weight, const float *bias, void *out,
                             long long rows, int channels, int ngroups, float eps, int dtype, void *stream) {
    if (!y || !z || !out) return SSD_ERR_INVALID_ARG;
    if (rows < 0 || channels < 1 || ngroups < 1 || channels % ngroups != 0 || !(eps >= 0.f)) return SSD_ERR_INVALID_ARG;
    if (dtype != SSD_F32 && dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
    if (channels / ngroups > ssd::kGnMaxGroup) return SSD_ERR_UNSUPPORTED;
    if (rows > (1LL << 40) || rows * (long long)ngroups > 8LL * 2147483647LL) return SSD_ERR_UNSUPPORTED;
    const size_t es = dtype == SSD_BF16 ? 2 : 4;
    if (!ssd::gn_aligned(y, es) || !ssd::gn_aligned(z, es) || !ssd::gn_aligned(out, es) ||
        (weight && !ssd::gn_aligned(weight, 4)) || (bias && !ssd::gn_aligned(bias, 4)))
        return SSD_ERR_INVALID_ARG;
    const size_t nbytes = es * (size_t)rows * channels;
    // out may be y itself (in place); it must not partly overlap y or overlap z
    if (nbytes && ((out != y && ssd::gn_overlap(out, nbytes, y, nbytes)) || ssd::gn_overlap(out, nbytes, z, nbytes)))
        return SSD_ERR_INVALID_ARG;
    if (rows == 0) return SSD_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // 16-byte vector accesses of y, z and out
    const bool vec_ok = ssd::gn_aligned(y, 16) && ssd::gn_aligned(z, 16) && ssd::gn_aligned(out, 16);
    const cudaError_t e =
        dtype == SSD_BF16
            ? ssd::launch_gate_norm<__nv_bfloat16>(y, z, weight, bias, out, rows, channels, ngroups, eps, vec_ok, st)
            : ssd::launch_gate_norm<float>(y, z, weight, bias, out, rows, channels, ngroups, eps, vec_ok, st);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
