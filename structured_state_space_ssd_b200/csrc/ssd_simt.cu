// ssd_simt.cu -- CUDA-core (fp32 FFMA) kernels of the SSD forward.
//
// These kernels follow the block decomposition of "Transformers are SSMs"
// (analysis page, section "The Block-Decomposition SSD Algorithm") one stage
// per kernel and serve every shape within the library's limits, in fp32 and
// bf16.  They are the path for fp32 inputs, whose tolerance the bf16 tensor
// cores cannot meet, and for shapes outside the tensor-core tile set.
//
// Log-space convention (all kernels): within chunk c, s[i] is the inclusive
// prefix sum of dt*A over the chunk's rows 0..i, so the product of decays
// a_{i+1} ... a_j is exp(s[j] - s[i]) and every exponent that is evaluated is
// a difference with a non-positive value for decaying inputs (never exp(-s)).
#include "ssd_common.cuh"

namespace ssd {

// ---------------------------------------------------------------------------
// Per-chunk inclusive prefix sums of dt*A (stage 0 partition + the exponents
// of the 1-semiseparable mask).  grid (nc, batch, ceil(H/32)), 256 threads: a
// block stages the [Q x 32] tile of dt for its heads with coalesced loads,
// then each warp scans one head's chunk: a sequential run over <= 8 elements per lane, then a
// shuffle scan of the lane totals.  Rows past the end of a short last chunk
// copy the last valid row, so s[Q-1] is always the chunk total.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) chunk_cumsum_kernel(const float *__restrict__ dt,
                                                           const float *__restrict__ A,
                                                           float *__restrict__ s, Shape sh) {
    extern __shared__ float tile[];  // [Q][33]
    const int c = blockIdx.x, b = blockIdx.y;
    const int t0 = c * sh.Q;
    const int len = min(sh.Q, sh.T - t0);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int E = (sh.Q + 31) >> 5;
    {
        const int h0 = blockIdx.z * 32;
        const int hn = min(32, sh.H - h0);
        // eight loads in flight per thread (rows i .. i+7*8 of one head column)
        for (int base = threadIdx.x; base < sh.Q * 32; base += 8 * blockDim.x) {
            float v[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int idx = base + r * blockDim.x;
                const int i = idx >> 5, hh = idx & 31;
                v[r] = (idx < sh.Q * 32 && i < len && hh < hn)
                           ? dt[((size_t)b * sh.T + t0 + i) * sh.H + h0 + hh] * A[h0 + hh]
                           : 0.f;
            }
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int idx = base + r * blockDim.x;
                if (idx < sh.Q * 32) tile[(idx >> 5) * 33 + (idx & 31)] = v[r];
            }
        }
        __syncthreads();
        for (int hh = warp; hh < hn; hh += nwarps) {
            float loc[8];
            float run = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int i = lane * E + e;
                if (e < E && i < sh.Q) run += tile[i * 33 + hh];
                loc[e] = run;
            }
            float incl = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            float excl = __shfl_up_sync(0xffffffffu, incl, 1);
            if (lane == 0) excl = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int i = lane * E + e;
                if (e < E && i < len) tile[i * 33 + hh] = loc[e] + excl;
            }
        }
        __syncthreads();
        // Rows past a short last chunk repeat the last valid row bit for bit, so
        // s[Q-1] is exactly s[len-1] and exp(s_end - s_last) is exactly 1 (a
        // reassociated sum could differ by one ulp, which is 8 at |s| ~ 1e8).
        for (int idx = threadIdx.x; idx < (sh.Q - len) * 32; idx += blockDim.x) {
            const int i = len + (idx >> 5), hh = idx & 31;
            tile[i * 33 + hh] = tile[(len - 1) * 33 + hh];
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < hn * sh.Q; idx += blockDim.x) {
            const int hh = idx / sh.Q, i = idx - hh * sh.Q;
            s[(((size_t)b * sh.H + h0 + hh) * sh.nc + c) * sh.Q + i] = tile[i * 33 + hh];
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Stage 2: chunk-final states from a zero start,
//   S_c[p][n] = sum_i exp(s_end - s_i) * x_i[p] * B_i[n].
// With from_start the weights are exp(s_i) instead (the decay from the chunk's
// start): the backward pass's chunk sums of dy_i C_i^T use this form.
// grid (nc, H, batch), 256 threads as 16 (n) x 16 (p); each thread owns an
// RP x RN register tile.  Rows are staged through shared memory 32 at a time.
// ---------------------------------------------------------------------------
template <typename T, int RP, int RN>
__global__ void __launch_bounds__(256) chunk_state_kernel(const T *__restrict__ x, const T *__restrict__ Bm,
                                                          const float *__restrict__ s, float *__restrict__ S,
                                                          Shape sh, bool from_start, bool vec) {
    extern __shared__ __align__(16) float smem[];
    float *Xs = smem;               // [32][P]
    float *Bs = smem + 32 * sh.P;   // [32][N]
    float *wr = Bs + 32 * sh.N;     // [32] decay weight of each row
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / sh.heads_per_group;
    const int t0 = c * sh.Q, len = min(sh.Q, sh.T - t0);
    const float *sc = s + (((size_t)b * sh.H + h) * sh.nc + c) * sh.Q;
    const float s_end = sc[sh.Q - 1];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[RP][RN];
#pragma unroll
    for (int r = 0; r < RP; ++r)
#pragma unroll
        for (int m = 0; m < RN; ++m) acc[r][m] = 0.f;

    for (int i0 = 0; i0 < len; i0 += 32) {
        // rows i0 .. i0+31 of x and B (16-byte loads when the rows allow), and each row's weight
        stage_rows<T>(Xs, sh.P, x + (((size_t)b * sh.T + t0 + i0) * sh.H + h) * sh.P, (size_t)sh.H * sh.P, 32,
                      len - i0, sh.P, sh.P, vec);
        stage_rows<T>(Bs, sh.N, Bm + (((size_t)b * sh.T + t0 + i0) * sh.G + g) * sh.N, (size_t)sh.G * sh.N, 32,
                      len - i0, sh.N, sh.N, vec);
        if (threadIdx.x < 32) {
            const int i = i0 + threadIdx.x;
            wr[threadIdx.x] = (i < len) ? expf(from_start ? sc[i] : s_end - sc[i]) : 0.f;
        }
        __syncthreads();
        for (int ii = 0; ii < 32; ++ii) {
            float xv[RP], bv[RN];
            const float wi = wr[ii];
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const int p = ty + 16 * r;
                xv[r] = (p < sh.P) ? Xs[ii * sh.P + p] * wi : 0.f;
            }
#pragma unroll
            for (int m = 0; m < RN; ++m) {
                const int n = tx + 16 * m;
                bv[m] = (n < sh.N) ? Bs[ii * sh.N + n] : 0.f;
            }
#pragma unroll
            for (int r = 0; r < RP; ++r)
#pragma unroll
                for (int m = 0; m < RN; ++m) acc[r][m] = fmaf(xv[r], bv[m], acc[r][m]);
        }
        __syncthreads();
    }
    float *out = S + (((size_t)b * sh.nc + c) * sh.H + h) * (size_t)sh.P * sh.N;
#pragma unroll
    for (int r = 0; r < RP; ++r) {
        const int p = ty + 16 * r;
#pragma unroll
        for (int m = 0; m < RN; ++m) {
            const int n = tx + 16 * m;
            if (p < sh.P && n < sh.N) out[(size_t)p * sh.N + n] = acc[r][m];
        }
    }
}

// ---------------------------------------------------------------------------
// Stage 3: the scalar recurrence between chunks, on all P*N channels,
//   S~_c = exp(s_end,c) * S~_{c-1} + S_c,   S~_{-1} = init_state (or 0).
// In place: slot c of S receives S~_{c-1}, the state entering chunk c; the
// last S~ goes to final_state.  grid (ceil(P*N/256), H, batch); the loads of
// up to 8 chunks are issued ahead of the dependent chain.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) state_passing_kernel(float *__restrict__ S, const float *__restrict__ s,
                                                            const float *__restrict__ init,
                                                            float *__restrict__ fin, Shape sh) {
    const int PN = sh.P * sh.N;
    const int e = blockIdx.x * 256 + threadIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    if (e >= PN) return;
    float run = init ? init[((size_t)b * sh.H + h) * PN + e] : 0.f;
    const float *sb = s + ((size_t)b * sh.H + h) * sh.nc * sh.Q;
    const size_t cstride = (size_t)sh.H * PN;
    float *base = S + ((size_t)b * sh.nc * sh.H + h) * PN + e;
    for (int c0 = 0; c0 < sh.nc; c0 += 8) {
        const int cn = min(8, sh.nc - c0);
        float loc[8], dec[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k < cn) {
                loc[k] = base[(size_t)(c0 + k) * cstride];
                dec[k] = expf(sb[(size_t)(c0 + k) * sh.Q + sh.Q - 1]);
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k < cn) {
                base[(size_t)(c0 + k) * cstride] = run;
                run = fmaf(dec[k], run, loc[k]);
            }
        }
    }
    if (fin) fin[((size_t)b * sh.H + h) * PN + e] = run;
}

// The same with four consecutive channels per thread (16-byte loads and stores), for P*N a multiple of 4
// and 16-byte aligned initial and final states: grid (ceil(P*N/1024), H, batch).
__global__ void __launch_bounds__(256) state_passing_vec_kernel(float *__restrict__ S, const float *__restrict__ s,
                                                                const float *__restrict__ init,
                                                                float *__restrict__ fin, Shape sh) {
    const int PN = sh.P * sh.N;
    const int e = (blockIdx.x * 256 + threadIdx.x) * 4;
    const int h = blockIdx.y, b = blockIdx.z;
    if (e >= PN) return;
    float4 run = init ? *reinterpret_cast<const float4 *>(init + ((size_t)b * sh.H + h) * PN + e)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    const float *sb = s + ((size_t)b * sh.H + h) * sh.nc * sh.Q;
    const size_t cstride = (size_t)sh.H * PN;
    float *base = S + ((size_t)b * sh.nc * sh.H + h) * PN + e;
    for (int c0 = 0; c0 < sh.nc; c0 += 8) {
        const int cn = min(8, sh.nc - c0);
        float4 loc[8];
        float dec[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k < cn) {
                loc[k] = *reinterpret_cast<const float4 *>(base + (size_t)(c0 + k) * cstride);
                dec[k] = expf(sb[(size_t)(c0 + k) * sh.Q + sh.Q - 1]);
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k < cn) {
                *reinterpret_cast<float4 *>(base + (size_t)(c0 + k) * cstride) = run;
                run = make_float4(fmaf(dec[k], run.x, loc[k].x), fmaf(dec[k], run.y, loc[k].y),
                                  fmaf(dec[k], run.z, loc[k].z), fmaf(dec[k], run.w, loc[k].w));
            }
        }
    }
    if (fin) *reinterpret_cast<float4 *>(fin + ((size_t)b * sh.H + h) * PN + e) = run;
}

// ---------------------------------------------------------------------------
// Stages 1, 4 and 5 fused, plus the D skip, for one 64-row tile of one chunk
// and one head:
//   y[j] = exp(s_j) C_j^T S~_{c-1}                       (stage 4)
//        + sum_{i<=j} exp(s_j - s_i) (C_j . B_i) x_i      (stage 1)
//        + D_h x_j.
// grid (nc * ceil(Q/64), H, batch), 256 threads as 16 (p) x 16 (rows); each
// thread owns 4 rows x RP columns.
// ---------------------------------------------------------------------------
template <typename T, int RP>
__global__ void __launch_bounds__(256) chunk_scan_kernel(const T *__restrict__ x, const T *__restrict__ Bm,
                                                         const T *__restrict__ Cm, const float *__restrict__ D,
                                                         const float *__restrict__ s,
                                                         const float *__restrict__ Sprev, T *__restrict__ y,
                                                         Shape sh) {
    extern __shared__ float smem[];
    const int NP = sh.N + 1;
    float *Cs = smem;              // [64][N+1]
    float *Bs = Cs + 64 * NP;      // [32][N+1]
    float *Xs = Bs + 32 * NP;      // [32][P]
    float *Ms = Xs + 32 * sh.P;    // [64][33]
    float *sj = Ms + 64 * 33;      // [64]
    float *si = sj + 64;           // [32]
    float *Ss = si + 32;           // [P][33]
    const int tiles = (sh.Q + 63) >> 6;
    const int c = blockIdx.x / tiles, jt = blockIdx.x - c * tiles;
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / sh.heads_per_group;
    const int t0 = c * sh.Q, len = min(sh.Q, sh.T - t0);
    const int j0 = jt * 64;
    if (j0 >= len) return;
    const int jn = min(64, len - j0);
    const float *sc = s + (((size_t)b * sh.H + h) * sh.nc + c) * sh.Q;

    for (int idx = threadIdx.x; idx < 64 * sh.N; idx += 256) {
        const int jj = idx / sh.N, n = idx - jj * sh.N;
        Cs[jj * NP + n] = (jj < jn) ? to_f32(Cm[(((size_t)b * sh.T + t0 + j0 + jj) * sh.G + g) * sh.N + n]) : 0.f;
    }
    if (threadIdx.x < 64) sj[threadIdx.x] = (threadIdx.x < jn) ? sc[j0 + threadIdx.x] : 0.f;
    __syncthreads();

    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][RP];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int k = 0; k < RP; ++k) acc[r][k] = 0.f;

    // stage 4: C_j^T S~_{c-1}, then the decay exp(s_j) from the chunk start
    const float *Sp = Sprev + (((size_t)b * sh.nc + c) * sh.H + h) * (size_t)sh.P * sh.N;
    for (int n0 = 0; n0 < sh.N; n0 += 32) {
        for (int idx = threadIdx.x; idx < sh.P * 32; idx += 256) {
            const int p = idx >> 5, nn = idx & 31;
            Ss[p * 33 + nn] = (n0 + nn < sh.N) ? Sp[(size_t)p * sh.N + n0 + nn] : 0.f;
        }
        __syncthreads();
        const int nlim = min(32, sh.N - n0);
        for (int nn = 0; nn < nlim; ++nn) {
            float cv[4], sv[RP];
#pragma unroll
            for (int r = 0; r < 4; ++r) cv[r] = Cs[(ty + 16 * r) * NP + n0 + nn];
#pragma unroll
            for (int k = 0; k < RP; ++k) {
                const int p = tx + 16 * k;
                sv[k] = (p < sh.P) ? Ss[p * 33 + nn] : 0.f;
            }
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int k = 0; k < RP; ++k) acc[r][k] = fmaf(cv[r], sv[k], acc[r][k]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const float e = expf(sj[ty + 16 * r]);
#pragma unroll
        for (int k = 0; k < RP; ++k) acc[r][k] *= e;
    }

    // stage 1: the masked quadratic form over columns i <= j of this chunk
    const int iend = j0 + jn;
    for (int i0 = 0; i0 < iend; i0 += 32) {
        for (int idx = threadIdx.x; idx < 32 * sh.N; idx += 256) {
            const int ii = idx / sh.N, n = idx - ii * sh.N, i = i0 + ii;
            Bs[ii * NP + n] = (i < iend) ? to_f32(Bm[(((size_t)b * sh.T + t0 + i) * sh.G + g) * sh.N + n]) : 0.f;
        }
        for (int idx = threadIdx.x; idx < 32 * sh.P; idx += 256) {
            const int ii = idx / sh.P, p = idx - ii * sh.P, i = i0 + ii;
            Xs[idx] = (i < iend) ? to_f32(x[(((size_t)b * sh.T + t0 + i) * sh.H + h) * sh.P + p]) : 0.f;
        }
        if (threadIdx.x < 32) si[threadIdx.x] = (i0 + threadIdx.x < iend) ? sc[i0 + threadIdx.x] : 0.f;
        __syncthreads();
        {
            const int jj = threadIdx.x >> 2, ib = (threadIdx.x & 3) * 8;
            float dot[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) dot[e] = 0.f;
            for (int n = 0; n < sh.N; ++n) {
                const float cv = Cs[jj * NP + n];
#pragma unroll
                for (int e = 0; e < 8; ++e) dot[e] = fmaf(cv, Bs[(ib + e) * NP + n], dot[e]);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int ii = ib + e, i = i0 + ii, j = j0 + jj;
                Ms[jj * 33 + ii] = (i <= j && jj < jn && i < iend) ? expf(sj[jj] - si[ii]) * dot[e] : 0.f;
            }
        }
        __syncthreads();
        for (int ii = 0; ii < 32; ++ii) {
            float mv[4], xv[RP];
#pragma unroll
            for (int r = 0; r < 4; ++r) mv[r] = Ms[(ty + 16 * r) * 33 + ii];
#pragma unroll
            for (int k = 0; k < RP; ++k) {
                const int p = tx + 16 * k;
                xv[k] = (p < sh.P) ? Xs[ii * sh.P + p] : 0.f;
            }
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int k = 0; k < RP; ++k) acc[r][k] = fmaf(mv[r], xv[k], acc[r][k]);
        }
        __syncthreads();
    }

    // stage 5 (the sum is already in acc) and the skip term
    const float Dh = D[h];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int jj = ty + 16 * r;
        if (jj >= jn) continue;
        const size_t row = (((size_t)b * sh.T + t0 + j0 + jj) * sh.H + h) * sh.P;
#pragma unroll
        for (int k = 0; k < RP; ++k) {
            const int p = tx + 16 * k;
            if (p < sh.P) y[row + p] = from_f32<T>(fmaf(Dh, to_f32(x[row + p]), acc[r][k]));
        }
    }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
static int pow2_at_least(int v) {
    int r = 1;
    while (r < v) r <<= 1;
    return r;
}

cudaError_t launch_chunk_cumsum(const float *dt, const float *A, float *s, const Shape &sh, cudaStream_t st) {
    const size_t smem = sizeof(float) * (size_t)sh.Q * 33;
    chunk_cumsum_kernel<<<dim3(sh.nc, sh.batch, (sh.H + 31) / 32), 256, smem, st>>>(dt, A, s, sh);
    return cudaGetLastError();
}

template <typename T, int RP, int RN>
static cudaError_t launch_state_rprn(const T *x, const T *B, const float *s, float *S, const Shape &sh,
                                     cudaStream_t st, bool from_start) {
    const size_t smem = sizeof(float) * (32 * (size_t)(sh.P + sh.N) + 32);
    auto k = chunk_state_kernel<T, RP, RN>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // 16-byte row loads: aligned tensors whose rows (P and N elements) are whole vectors
    constexpr int VE = 16 / (int)sizeof(T);
    const bool vec = reinterpret_cast<uintptr_t>(x) % 16 == 0 && reinterpret_cast<uintptr_t>(B) % 16 == 0 &&
                     sh.P % VE == 0 && sh.N % VE == 0;
    k<<<dim3(sh.nc, sh.H, sh.batch), 256, smem, st>>>(x, B, s, S, sh, from_start, vec);
    return cudaGetLastError();
}

template <typename T, int RP>
static cudaError_t launch_state_rp(const T *x, const T *B, const float *s, float *S, const Shape &sh,
                                   cudaStream_t st, bool from_start) {
    switch (pow2_at_least((sh.N + 15) / 16)) {
        case 1: return launch_state_rprn<T, RP, 1>(x, B, s, S, sh, st, from_start);
        case 2: return launch_state_rprn<T, RP, 2>(x, B, s, S, sh, st, from_start);
        case 4: return launch_state_rprn<T, RP, 4>(x, B, s, S, sh, st, from_start);
        case 8: return launch_state_rprn<T, RP, 8>(x, B, s, S, sh, st, from_start);
        default: return launch_state_rprn<T, RP, 16>(x, B, s, S, sh, st, from_start);
    }
}

template <typename T>
cudaError_t launch_chunk_state(const T *x, const T *B, const float *s, float *S, const Shape &sh, cudaStream_t st,
                               bool from_start) {
    switch (pow2_at_least((sh.P + 15) / 16)) {
        case 1: return launch_state_rp<T, 1>(x, B, s, S, sh, st, from_start);
        case 2: return launch_state_rp<T, 2>(x, B, s, S, sh, st, from_start);
        case 4: return launch_state_rp<T, 4>(x, B, s, S, sh, st, from_start);
        default: return launch_state_rp<T, 8>(x, B, s, S, sh, st, from_start);
    }
}

cudaError_t launch_state_passing(float *S, const float *s, const float *init, float *fin, const Shape &sh,
                                 cudaStream_t st) {
    const int PN = sh.P * sh.N;
    if (PN % 4 == 0 && reinterpret_cast<uintptr_t>(init) % 16 == 0 && reinterpret_cast<uintptr_t>(fin) % 16 == 0)
        state_passing_vec_kernel<<<dim3((PN + 1023) / 1024, sh.H, sh.batch), 256, 0, st>>>(S, s, init, fin, sh);
    else
        state_passing_kernel<<<dim3((PN + 255) / 256, sh.H, sh.batch), 256, 0, st>>>(S, s, init, fin, sh);
    return cudaGetLastError();
}

template <typename T, int RP>
static cudaError_t launch_scan_rp(const T *x, const T *B, const T *C, const float *D, const float *s,
                                  const float *Sprev, T *y, const Shape &sh, cudaStream_t st) {
    const size_t smem = sizeof(float) * ((size_t)96 * (sh.N + 1) + 32 * sh.P + 64 * 33 + 96 + (size_t)sh.P * 33);
    auto k = chunk_scan_kernel<T, RP>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int tiles = (sh.Q + 63) / 64;
    k<<<dim3(sh.nc * tiles, sh.H, sh.batch), 256, smem, st>>>(x, B, C, D, s, Sprev, y, sh);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_chunk_scan(const T *x, const T *B, const T *C, const float *D, const float *s,
                              const float *Sprev, T *y, const Shape &sh, cudaStream_t st) {
    switch (pow2_at_least((sh.P + 15) / 16)) {
        case 1: return launch_scan_rp<T, 1>(x, B, C, D, s, Sprev, y, sh, st);
        case 2: return launch_scan_rp<T, 2>(x, B, C, D, s, Sprev, y, sh, st);
        case 4: return launch_scan_rp<T, 4>(x, B, C, D, s, Sprev, y, sh, st);
        default: return launch_scan_rp<T, 8>(x, B, C, D, s, Sprev, y, sh, st);
    }
}

template cudaError_t launch_chunk_state<float>(const float *, const float *, const float *, float *, const Shape &,
                                               cudaStream_t, bool);
template cudaError_t launch_chunk_state<__nv_bfloat16>(const __nv_bfloat16 *, const __nv_bfloat16 *, const float *,
                                                       float *, const Shape &, cudaStream_t, bool);
template cudaError_t launch_chunk_scan<float>(const float *, const float *, const float *, const float *,
                                              const float *, const float *, float *, const Shape &, cudaStream_t);
template cudaError_t launch_chunk_scan<__nv_bfloat16>(const __nv_bfloat16 *, const __nv_bfloat16 *,
                                                      const __nv_bfloat16 *, const float *, const float *,
                                                      const float *, __nv_bfloat16 *, const Shape &, cudaStream_t);

}  // namespace ssd
