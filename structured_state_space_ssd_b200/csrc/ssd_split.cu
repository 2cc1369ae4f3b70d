// ssd_split.cu -- a sequence split into contiguous shards that exchange only states.
//
// Sequence (context) parallelism: workers process contiguous shards of the
// sequence and pass recurrent states between them, with communication linear
// in the number of workers (the paper's claim summary on its reproduction
// page; the "Transformers are SSMs" analysis page, section "The
// Block-Decomposition SSD Algorithm", stages 3 and 4, is the same
// decomposition one level up: shards play the role of chunks).
//
// With shard k covering tokens [t_k, t_{k+1}) and sigma_t the inclusive sum of
// dt_u * A_h from t_k to t, the forward of the shard from a zero state gives
// y0 and fin0, and with the state S_in entering the shard
//
//     y_t = y0_t + exp(sigma_t) S_in C_t        fin = fin0 + exp(sigma_end) S_in
//     S_in(k) = fin(k-1),  S_in(0) = init_state (or 0)
//
// so every shard can run its forward at once, exchange (fin0, sigma_end) once,
// fold the earlier shards' pairs into its S_in, and correct its own outputs.
// Three kernels: the per-token log-decay prefix of a shard, the fold, and the
// output correction (a [T x N] x [N x P] product per head, on the CUDA cores).
#include "ssd_common.cuh"

namespace ssd {

namespace {

constexpr int kScanThreads = 256;

// sig[b][h][t] = sum_{u <= t} dt[b][u][h] * A[h] over the shard; total[b][h] = sig at the last token.
// One block per (b, h): each thread sums a contiguous run of tokens, a block scan of the run totals
// gives every run its offset, and a second pass writes the prefix.
__global__ void __launch_bounds__(kScanThreads)
    split_logdecay_kernel(const float *__restrict__ dt, const float *__restrict__ A, float *__restrict__ sig,
                          float *__restrict__ total, int T, int H) {
    __shared__ float part[kScanThreads];
    const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const float a = A[h];
    const int run = (T + kScanThreads - 1) / kScanThreads;
    const int t0 = tid * run, t1 = min(T, t0 + run);
    const float *d = dt + (size_t)b * T * H + h;
    float s = 0.f;
    for (int t = t0; t < t1; ++t) s += d[(size_t)t * H] * a;
    part[tid] = s;
    __syncthreads();
    // inclusive Hillis-Steele scan of the run totals
    for (int o = 1; o < kScanThreads; o <<= 1) {
        const float v = tid >= o ? part[tid - o] : 0.f;
        __syncthreads();
        part[tid] += v;
        __syncthreads();
    }
    float acc = tid > 0 ? part[tid - 1] : 0.f;
    float *out = sig + ((size_t)b * H + h) * T;
    for (int t = t0; t < t1; ++t) {
        acc += d[(size_t)t * H] * a;
        out[t] = acc;
    }
    if (tid == kScanThreads - 1) total[(size_t)b * H + h] = part[kScanThreads - 1];
}

// S_in(k) = fold over shards j < k of S <- exp(total_j) S + fin0_j, from S = init (or 0); and the shard's
// own final state fin0_k + exp(total_k) S_in(k).  One thread per state element.
__global__ void split_combine_kernel(const float *__restrict__ fin0_all, const float *__restrict__ total_all,
                                     const float *__restrict__ init, int k, float *__restrict__ s_in,
                                     float *__restrict__ fin_out, long long elems, int per_bh, int bh_count) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= elems) return;
    const int bh = (int)(i / per_bh);
    float s = init ? init[i] : 0.f;
    for (int j = 0; j < k; ++j) s = fmaf(expf(total_all[(size_t)j * bh_count + bh]), s, fin0_all[(size_t)j * elems + i]);
    s_in[i] = s;
    if (fin_out)
        fin_out[i] = fmaf(expf(total_all[(size_t)k * bh_count + bh]), s, fin0_all[(size_t)k * elems + i]);
}

// y[b][t][h][p] += exp(sig[b][h][t]) * sum_n S_in[b][h][p][n] C[b][t][g][n].  Block = (b, h, 32 tokens),
// 256 threads: S_in and the tokens' C rows in shared memory (rows padded by one float), 8 threads per
// token, each accumulating every eighth p.
constexpr int kCorrTokens = 32;

template <typename T>
__global__ void __launch_bounds__(256)
    split_correct_kernel(T *__restrict__ y, const T *__restrict__ C, const float *__restrict__ sig,
                         const float *__restrict__ s_in, int Tn, int H, int P, int G, int N) {
    extern __shared__ float sm[];
    const int ld = N + 1;                 // padded rows: the 8 p (or 4 tokens) a warp reads hit 8 banks
    float *S = sm;                        // [P][N + 1]
    float *Cs = sm + (size_t)P * ld;      // [kCorrTokens][N + 1]
    const int h = blockIdx.y, b = blockIdx.z, t0 = blockIdx.x * kCorrTokens;
    const int g = h / (H / G);
    const size_t bh = (size_t)b * H + h;
    for (int i = threadIdx.x; i < P * N; i += blockDim.x) S[(i / N) * ld + i % N] = s_in[bh * P * N + i];
    for (int i = threadIdx.x; i < kCorrTokens * N; i += blockDim.x) {
        const int tt = i / N, n = i % N, t = t0 + tt;
        Cs[tt * ld + n] = t < Tn ? to_f32(C[(((size_t)b * Tn + t) * G + g) * N + n]) : 0.f;
    }
    __syncthreads();
    const int tt = threadIdx.x >> 3, lane8 = threadIdx.x & 7, t = t0 + tt;  // 8 threads per token
    if (t >= Tn) return;
    const float e = expf(sig[bh * Tn + t]);
    const float *c = Cs + (size_t)tt * ld;
    T *yr = y + (((size_t)b * Tn + t) * H + h) * P;
    for (int p = lane8; p < P; p += 8) {
        const float *srow = S + (size_t)p * ld;
        float acc = 0.f;
        for (int n = 0; n < N; ++n) acc = fmaf(srow[n], c[n], acc);
        yr[p] = from_f32<T>(to_f32(yr[p]) + e * acc);
    }
}

bool sp_aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

}  // namespace ssd

extern "C" int ssd_split_logdecay(const float *dt, const float *A, float *sig, float *total, int batch, int T, int H,
                                  void *stream) {
    if (!dt || !A || !sig || !total || batch < 1 || T < 1 || H < 1) return SSD_ERR_INVALID_ARG;
    if (batch > 65535) return SSD_ERR_UNSUPPORTED;
    if (!ssd::sp_aligned(dt, 4) || !ssd::sp_aligned(A, 4) || !ssd::sp_aligned(sig, 4) || !ssd::sp_aligned(total, 4))
        return SSD_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    ssd::split_logdecay_kernel<<<dim3(H, batch), ssd::kScanThreads, 0, st>>>(dt, A, sig, total, T, H);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

extern "C" int ssd_split_combine(const float *fin0_all, const float *total_all, const float *init_state, int k,
                                 int shards, float *s_in, float *final_state, int batch, int H, int P, int N,
                                 void *stream) {
    if (!fin0_all || !total_all || !s_in || shards < 1 || k < 0 || k >= shards) return SSD_ERR_INVALID_ARG;
    if (batch < 1 || H < 1 || P < 1 || N < 1) return SSD_ERR_INVALID_ARG;
    const long long elems = (long long)batch * H * P * N;
    if (elems > (1LL << 40)) return SSD_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int threads = 256;
    ssd::split_combine_kernel<<<(unsigned)((elems + threads - 1) / threads), threads, 0, st>>>(
        fin0_all, total_all, init_state, k, s_in, final_state, elems, P * N, batch * H);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

extern "C" int ssd_split_correct(void *y, const void *C, const float *sig, const float *s_in, int batch, int T, int H,
                                 int P, int G, int N, int dtype, void *stream) {
    if (!y || !C || !sig || !s_in || batch < 1 || T < 0 || H < 1 || P < 1 || G < 1 || N < 1 || H % G != 0)
        return SSD_ERR_INVALID_ARG;
    if (dtype != SSD_F32 && dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
    if (T == 0) return SSD_OK;
    const size_t smem = sizeof(float) * ((size_t)P + ssd::kCorrTokens) * (N + 1);
    if (P > 128 || N > 256 || batch > 65535 || H > 65535 || smem > 227 * 1024) return SSD_ERR_UNSUPPORTED;
    const size_t es = dtype == SSD_BF16 ? 2 : 4;
    if (!ssd::sp_aligned(y, es) || !ssd::sp_aligned(C, es) || !ssd::sp_aligned(sig, 4) || !ssd::sp_aligned(s_in, 4))
        return SSD_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const dim3 grid((T + ssd::kCorrTokens - 1) / ssd::kCorrTokens, H, batch);
    cudaError_t e;
    if (dtype == SSD_BF16) {
        e = cudaFuncSetAttribute(ssd::split_correct_kernel<__nv_bfloat16>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess)
            ssd::split_correct_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(
                static_cast<__nv_bfloat16 *>(y), static_cast<const __nv_bfloat16 *>(C), sig, s_in, T, H, P, G, N);
    } else {
        e = cudaFuncSetAttribute(ssd::split_correct_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e == cudaSuccess)
            ssd::split_correct_kernel<float><<<grid, 256, smem, st>>>(static_cast<float *>(y),
                                                                      static_cast<const float *>(C), sig, s_in, T, H,
                                                                      P, G, N);
    }
    if (e != cudaSuccess) return SSD_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
