// ssd_bwd.cu -- the SSD layer backward on the CUDA cores: gradients of
// (y, final_state) with respect to x, dt, A, B, C, D and the initial state.
//
// The pages give the forward only ("Transformers are SSMs", analysis page,
// section "The Block-Decomposition SSD Algorithm"); the backward here is the
// gradient of that function, organised by the same chunk decomposition.  With
// s_i the inclusive log-decay prefix of a chunk (s_end its last value), Hin_c
// the state entering chunk c and dHout_c the gradient arriving at the state
// that leaves it:
//
//   dHout_{nc-1} = dfinal,   dHout_{c-1} = exp(s_end,c) dHout_c + sum_i exp(s_i) dy_i C_i^T
//   dinit = dHout_{-1}
//   dx_r  = exp(s_end - s_r) dHout_c B_r + sum_{i>=r} exp(s_i - s_r) (B_r . C_i) dy_i + D_h dy_r
//   dB_r  = sum over heads of [exp(s_end - s_r) x_r^T dHout_c + sum_{i>=r} exp(s_i - s_r) (x_r . dy_i) C_i]
//   dC_r  = sum over heads of [exp(s_r) dy_r^T Hin_c + sum_{i<=r} exp(s_r - s_i) (dy_r . x_i) B_i]
//
// and the decays enter through the per-token gradient of the running
// log-decay sigma_t = sum_{u<=t} dt_u A_h of the whole sequence:
//
//   dsigma_t = C_t . dC_t^(h) - B_t . dB_t^(h)   (+ <dfinal, final> at the last token)
//   d(dt_u A_h) = sum_{t>=u} dsigma_t,   ddt_u = A_h d(dt_u A_h),   dA_h = sum dt_u d(dt_u A_h)
//
// where dB^(h), dC^(h) are one head's terms before the sum over its group.
// The three products above share one masked-scan kernel (the forward's
// chunk_scan shape with the roles of its operands exchanged); the chunk sums
// and the forward states reuse the forward's CUDA-core kernels.  Every
// reduction runs in a fixed order: results are bitwise reproducible.
#include <algorithm>

#include "ssd_common.cuh"

namespace ssd {
cudaError_t launch_chunk_cumsum(const float *dt, const float *A, float *s, const Shape &sh, cudaStream_t st);
template <typename T>
cudaError_t launch_chunk_state(const T *x, const T *B, const float *s, float *S, const Shape &sh, cudaStream_t st,
                               bool from_start);
cudaError_t launch_state_passing(float *S, const float *s, const float *init, float *fin, const Shape &sh,
                                 cudaStream_t st);

// The masked scans on the tensor cores (ssd_bwd_tc.cu); which of the three run there: bit 0 dx, bit 1 the
// per-head dB terms, bit 2 the per-head dC terms.
bool scan_tc_supported(const Shape &sh, int dtype);
// With `part` given, the dB or dC scan sums its terms over each group's heads instead of storing them;
// launch_head_sum_reduce then forms dB, dC and dsigma from both scans' partial results.
cudaError_t launch_masked_scan_tc(const void *R, int r_head, const void *K, int k_head, const void *V, int v_head,
                                  int KD, int W, bool anti, const float *St, int st_kw, const float *D, void *out,
                                  bool out_bf16, const float *s, int *status, const Shape &sh, cudaStream_t st,
                                  const void *dotv = nullptr, float *dotp = nullptr, float *part = nullptr);
cudaError_t launch_head_sum_reduce(const float *partB, const float *dotB, const float *partC, const float *dotC,
                                   void *dB, void *dC, float *dsig, const Shape &sh, cudaStream_t st);
constexpr int kScanTcRoles = 7;
// chunk states on the tensor cores (ssd_bwd_tc.cu): bf16, P = 64, N = 128, Q in {128, 256}
bool chunk_state_tc_supported(const Shape &sh, int dtype);
cudaError_t launch_chunk_state_tc(const void *x, const void *B, const float *s, float *S, bool from_start,
                                  int *status, const Shape &sh, cudaStream_t st);

namespace {

// ---------------------------------------------------------------------------
// Workspace of one backward call (all offsets 256-byte aligned).
// ---------------------------------------------------------------------------
// The dD dot products over a sequence run in this many token slices (more blocks in flight), each with
// its own fp64 partial; the parameter sum adds them in a fixed order.
constexpr int kDdSlices = 4;

struct BwdWorkspace {
    size_t status_off;  // int status word of the tensor-core scans' bounded waits (cleared per call)
    size_t s_off;     // float s[batch][H][nc][Q]
    size_t hin_off;   // float Hin[batch][nc][H][P][N]: chunk states, then the state entering each chunk
    size_t gout_off;  // float G[batch][nc][H][P][N]: chunk sums of dy C^T, then dHout of each chunk
    size_t fin_off;   // float final[batch][H][P][N]
    size_t dbh_off;   // float dB^(h)[batch][T][H][N], or the dB scan's head sums (bwd_sum_bytes)
    size_t dch_off;   // float dC^(h)[batch][T][H][N], or the dC scan's head sums
    size_t dsig_off;  // float dsigma[batch][H][T]
    size_t pa_off;    // double dA partial[batch][H]
    size_t pd_off;    // double dD partial[kDdSlices][batch][H] (one per quarter of the tokens)
    size_t total;
};

BwdWorkspace bwd_layout(const Shape &s) {
    BwdWorkspace w;
    const size_t bh = (size_t)s.batch * s.H, PN = (size_t)s.P * s.N;
    const size_t states = sizeof(float) * (size_t)s.batch * s.nc * s.H * PN;
    const size_t perhead = std::max(sizeof(float) * (size_t)s.batch * s.T * s.H * s.N, bwd_sum_bytes(s));
    size_t off = 0;
    w.status_off = off;
    off = 256;
    w.s_off = off;
    off = align256(off + sizeof(float) * bh * s.nc * s.Q);
    w.hin_off = off;
    off = align256(off + states);
    w.gout_off = off;
    off = align256(off + states);
    w.fin_off = off;
    off = align256(off + sizeof(float) * bh * PN);
    w.dbh_off = off;
    off = align256(off + perhead);
    w.dch_off = off;
    off = align256(off + perhead);
    w.dsig_off = off;
    off = align256(off + sizeof(float) * bh * s.T);
    w.pa_off = off;
    off = align256(off + sizeof(double) * bh);
    w.pd_off = off;
    off = align256(off + sizeof(double) * kDdSlices * bh);
    w.total = off;
    return w;
}

// ---------------------------------------------------------------------------
// Reverse state passing, in place on the chunk sums G_c = sum_i exp(s_i) dy_i C_i^T:
// slot c receives dHout_c, and dinit (if requested) receives dHout_{-1}.
// grid (ceil(P*N/256), H, batch); the loads of up to 8 chunks go out ahead of
// the dependent chain, as in the forward's state passing.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) state_passing_bwd_kernel(float *__restrict__ Gs, const float *__restrict__ s,
                                                                const float *__restrict__ dfin,
                                                                float *__restrict__ dinit, Shape sh) {
    const int PN = sh.P * sh.N;
    const int e = blockIdx.x * 256 + threadIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    if (e >= PN) return;
    float run = dfin ? dfin[((size_t)b * sh.H + h) * PN + e] : 0.f;
    const float *sb = s + ((size_t)b * sh.H + h) * sh.nc * sh.Q;
    const size_t cstride = (size_t)sh.H * PN;
    float *base = Gs + ((size_t)b * sh.nc * sh.H + h) * PN + e;
    for (int cend = sh.nc; cend > 0; cend -= 8) {
        const int cn = min(8, cend), c0 = cend - cn;
        float loc[8], dec[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (k < cn) {
                loc[k] = base[(size_t)(c0 + k) * cstride];
                dec[k] = expf(sb[(size_t)(c0 + k) * sh.Q + sh.Q - 1]);
            }
        }
#pragma unroll
        for (int k = 7; k >= 0; --k) {
            if (k < cn) {
                base[(size_t)(c0 + k) * cstride] = run;
                run = fmaf(dec[k], run, loc[k]);
            }
        }
    }
    if (dinit) dinit[((size_t)b * sh.H + h) * PN + e] = run;
}

// The same with four consecutive channels per thread (16-byte loads and stores), for P*N a multiple of 4
// and 16-byte aligned dfin and dinit: grid (ceil(P*N/1024), H, batch).
__global__ void __launch_bounds__(256) state_passing_bwd_vec_kernel(float *__restrict__ Gs,
                                                                    const float *__restrict__ s,
                                                                    const float *__restrict__ dfin,
                                                                    float *__restrict__ dinit, Shape sh) {
    const int PN = sh.P * sh.N;
    const int e = (blockIdx.x * 256 + threadIdx.x) * 4;
    const int h = blockIdx.y, b = blockIdx.z;
    if (e >= PN) return;
    float4 run = dfin ? *reinterpret_cast<const float4 *>(dfin + ((size_t)b * sh.H + h) * PN + e)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    const float *sb = s + ((size_t)b * sh.H + h) * sh.nc * sh.Q;
    const size_t cstride = (size_t)sh.H * PN;
    float *base = Gs + ((size_t)b * sh.nc * sh.H + h) * PN + e;
    for (int cend = sh.nc; cend > 0; cend -= 8) {
        const int cn = min(8, cend), c0 = cend - cn;
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
        for (int k = 7; k >= 0; --k) {
            if (k < cn) {
                *reinterpret_cast<float4 *>(base + (size_t)(c0 + k) * cstride) = run;
                run = make_float4(fmaf(dec[k], run.x, loc[k].x), fmaf(dec[k], run.y, loc[k].y),
                                  fmaf(dec[k], run.z, loc[k].z), fmaf(dec[k], run.w, loc[k].w));
            }
        }
    }
    if (dinit) *reinterpret_cast<float4 *>(dinit + ((size_t)b * sh.H + h) * PN + e) = run;
}

// ---------------------------------------------------------------------------
// Masked scan over one chunk, one head and a 64-row tile:
//
//   out_r[w] = e_r * sum_k R_r[k] St[k][w]
//            + sum_{i in chunk, i >= r (kAnti) or i <= r} exp(+-(s_i - s_r)) (R_r . K_i) V_i[w]
//            + D_h V_r[w]                                          (when D is given)
//
// with e_r = exp(s_end - s_r) (kAnti: the state arrives at the chunk's end)
// or exp(s_r) (the state enters at its start).  Operands are rows of
// [batch][T][*] tensors: R and K have KD columns, V has W; each is either a
// head's slice (row length H*KD or H*W) or its group's (G*KD or G*W).  St is
// the [P][N] state of the (batch, chunk, head), read as [W][KD] or [KD][W].
// grid (nc * ceil(Q/64), H, batch), 256 threads.
//
// Shared memory, fp32 (KD4 = KD rounded up to 4; KP = KD4 + 4 keeps rows
// 16-byte aligned and puts eight consecutive rows on distinct bank quads;
// W64 = 64 RV >= W; SW = W64 + 4):
//   Rs [64][KP] the tile's rows of R     Ks [32][KP]  32 columns' rows of K
//   Vs [32][W64] their rows of V         Ss [32][SW]  32 contraction rows of the state
//   Ms [64][36] the masked weights of the 64 x 32 block;  sr [64], sc [32] prefix sums
// The output belongs to 16 (tx) x 16 (ty) threads: rows ty + 16 rr (rr < 4),
// columns 64 v + 4 tx + e (v < RV, e < 4), read as float4 rows of V and of the
// state.  The 64 x 32 dot products belong to 32 (rg) x 8 (cg) threads: rows
// rg + 32 p (p < 2), columns cg + 8 q (q < 4), float4 along the contraction.
// Every shared-memory operand is then used by at least two FMAs per load.
// ---------------------------------------------------------------------------
struct ScanArgs {
    const void *R, *K, *V;
    int r_head, k_head, v_head;  // 1: the head's slice, 0: the group's
    const float *St;             // [batch][nc][H][P*N]
    int st_kw;                   // 1: St is [KD][W], 0: [W][KD]
    int KD, W;
    const float *D;              // skip factor per head, or null
    void *out;                   // [batch][T][H][W]
    int vec;                     // R, K, V rows load as 16-byte vectors (aligned, KD and W multiples of it)
    int st_vec;                  // the state loads as float4 (its rows' lengths multiples of 4)
};

constexpr int kMsLd = 36;  // row length of Ms (32 columns, padded to keep float4 rows aligned)

// 16-byte asynchronous copy global -> shared (zero-filled when src_bytes is 0), and its group fences.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

template <typename T, typename TO, int RV, bool kAnti>
__global__ void __launch_bounds__(256) masked_scan_kernel(ScanArgs a, const float *__restrict__ s, Shape sh) {
    extern __shared__ __align__(16) float smem[];
    const int KD = a.KD, W = a.W;
    const int KD4 = (KD + 3) & ~3, KP = KD4 + 4;
    constexpr int W64 = 64 * RV, SW = W64 + 4;
    float *Rs = smem;              // [64][KP]
    float *Ks = Rs + 64 * KP;      // [32][KP]
    float *Vs = Ks + 32 * KP;      // [32][W64]
    float *Ss = Vs + 32 * W64;     // [32][SW]
    float *Ms = Ss + 32 * SW;      // [64][kMsLd]
    float *sr = Ms + 64 * kMsLd;   // [64]
    float *sc = sr + 64;           // [32]
    float *sq = sc + 32;           // [kMaxQ]: the chunk's prefix sums
    T *KsRaw = reinterpret_cast<T *>(sq + kMaxQ);  // [32][KD] next column tile as copied (vec only)
    T *VsRaw = KsRaw + 32 * KD;                    // [32][W]
    const int tiles = (sh.Q + 63) >> 6;
    const int c = blockIdx.x / tiles, jt = blockIdx.x - c * tiles;
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / sh.heads_per_group;
    const int t0 = c * sh.Q, len = min(sh.Q, sh.T - t0);
    const int j0 = jt * 64;
    if (j0 >= len) return;
    const int jn = min(64, len - j0);
    const float *sch = s + (((size_t)b * sh.H + h) * sh.nc + c) * sh.Q;
    const T *Rp = static_cast<const T *>(a.R);
    const T *Kp = static_cast<const T *>(a.K);
    const T *Vp = static_cast<const T *>(a.V);
    const size_t r_ld = (size_t)(a.r_head ? sh.H : sh.G) * KD, r_off = (size_t)(a.r_head ? h : g) * KD;
    const size_t k_ld = (size_t)(a.k_head ? sh.H : sh.G) * KD, k_off = (size_t)(a.k_head ? h : g) * KD;
    const size_t v_ld = (size_t)(a.v_head ? sh.H : sh.G) * W, v_off = (size_t)(a.v_head ? h : g) * W;
    const size_t row0 = (size_t)b * sh.T + t0;  // token index of the chunk's first row

    stage_rows<T>(Rs, KP, Rp + (row0 + j0) * r_ld + r_off, r_ld, 64, jn, KD, KD4, a.vec);
    if (threadIdx.x < 64) sr[threadIdx.x] = (threadIdx.x < jn) ? sch[j0 + threadIdx.x] : 0.f;
    for (int i = threadIdx.x; i < sh.Q; i += 256) sq[i] = sch[i];
    __syncthreads();

    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][RV][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int v = 0; v < RV; ++v)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[r][v][e] = 0.f;

    // the state term, 32 of the KD contraction indices at a time
    const float *Sp = a.St + (((size_t)b * sh.nc + c) * sh.H + h) * (size_t)sh.P * sh.N;
    for (int k0 = 0; k0 < KD; k0 += 32) {
        if (a.st_kw) {  // [KD][W]: rows k0.. of the state, lanes along w
            stage_rows<float>(Ss, SW, Sp + (size_t)k0 * W, W, 32, KD - k0, W, W64, a.st_vec);
        } else if (a.st_vec) {  // [W][KD], KD a multiple of 4: float4 along k, stored transposed
            const int total = W64 * 8;  // (row w, quad of k) pairs of the slab
            for (int base = threadIdx.x; base < total; base += 4 * 256) {
                float4 u[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int idx = base + q * 256, w = idx >> 3, k = k0 + 4 * (idx & 7);
                    u[q] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (idx < total && w < W && k < KD)
                        u[q] = *reinterpret_cast<const float4 *>(Sp + (size_t)w * KD + k);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int idx = base + q * 256, w = idx >> 3, kk = 4 * (idx & 7);
                    if (idx < total) {
                        Ss[kk * SW + w] = u[q].x;
                        Ss[(kk + 1) * SW + w] = u[q].y;
                        Ss[(kk + 2) * SW + w] = u[q].z;
                        Ss[(kk + 3) * SW + w] = u[q].w;
                    }
                }
            }
        } else {        // [W][KD]: a warp reads 8 consecutive k of 4 rows
            for (int idx = threadIdx.x; idx < 32 * W64; idx += 256) {
                const int lane = idx & 31, grp = idx >> 5;
                const int kk = (lane & 7) + 8 * (grp & 3), w = (lane >> 3) + 4 * (grp >> 2), k = k0 + kk;
                Ss[kk * SW + w] = (k < KD && w < W) ? Sp[(size_t)w * KD + k] : 0.f;
            }
        }
        __syncthreads();
        const int klim = min(32, KD - k0);
        for (int kk = 0; kk < klim; ++kk) {
            float rv[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) rv[r] = Rs[(ty + 16 * r) * KP + k0 + kk];
#pragma unroll
            for (int v = 0; v < RV; ++v) {
                const float4 sv = *reinterpret_cast<const float4 *>(Ss + kk * SW + 64 * v + 4 * tx);
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    acc[r][v][0] = fmaf(rv[r], sv.x, acc[r][v][0]);
                    acc[r][v][1] = fmaf(rv[r], sv.y, acc[r][v][1]);
                    acc[r][v][2] = fmaf(rv[r], sv.z, acc[r][v][2]);
                    acc[r][v][3] = fmaf(rv[r], sv.w, acc[r][v][3]);
                }
            }
        }
        __syncthreads();
    }
    {
        const float s_end = sch[sh.Q - 1];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const float sj = sr[ty + 16 * r];
            const float e = kAnti ? expf(s_end - sj) : expf(sj);
#pragma unroll
            for (int v = 0; v < RV; ++v)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[r][v][q] *= e;
        }
    }

    // the masked quadratic term over the chunk's other rows
    const int ibeg = kAnti ? j0 : 0;
    const int iend = kAnti ? len : j0 + jn;
    const int rg = threadIdx.x >> 3, cg = threadIdx.x & 7;
    // With 16-byte rows the next column tile is copied asynchronously (raw, into KsRaw / VsRaw) while
    // this one's products run, then widened to fp32 in shared memory.
    constexpr int VE = 16 / (int)sizeof(T);
    const bool pipe = a.vec;
    auto issue = [&](int i0n) {
        const int valid = iend - i0n, kcr = KD / VE, vcr = W / VE;
        for (int idx = threadIdx.x; idx < 32 * kcr; idx += 256) {
            const int r = idx / kcr, kc = idx - r * kcr;
            const bool ok = r < valid;
            cp_async16(KsRaw + r * KD + kc * VE, ok ? Kp + (row0 + i0n + r) * k_ld + k_off + kc * VE : Kp, ok ? 16 : 0);
        }
        for (int idx = threadIdx.x; idx < 32 * vcr; idx += 256) {
            const int r = idx / vcr, vc = idx - r * vcr;
            const bool ok = r < valid;
            cp_async16(VsRaw + r * W + vc * VE, ok ? Vp + (row0 + i0n + r) * v_ld + v_off + vc * VE : Vp, ok ? 16 : 0);
        }
        cp_async_commit();
    };
    if (pipe) {
        for (int idx = threadIdx.x; idx < 32 * (W64 - W); idx += 256) {  // padding columns stay zero
            const int r = idx / (W64 - W);
            Vs[r * W64 + W + (idx - r * (W64 - W))] = 0.f;
        }
        if (ibeg < iend) issue(ibeg);
    }
    for (int i0 = ibeg; i0 < iend; i0 += 32) {
        if (pipe) {
            cp_async_wait_all();
            __syncthreads();
            const int kcr = KD / VE, vcr = W / VE;
            for (int idx = threadIdx.x; idx < 32 * kcr; idx += 256) {
                const int r = idx / kcr, kc = idx - r * kcr;
                float f[VE];
                unpack16(*reinterpret_cast<const uint4 *>(KsRaw + r * KD + kc * VE), f, T());
                float4 *d = reinterpret_cast<float4 *>(Ks + r * KP + kc * VE);
#pragma unroll
                for (int e = 0; e < VE / 4; ++e) d[e] = make_float4(f[4 * e], f[4 * e + 1], f[4 * e + 2], f[4 * e + 3]);
            }
            for (int idx = threadIdx.x; idx < 32 * vcr; idx += 256) {
                const int r = idx / vcr, vc = idx - r * vcr;
                float f[VE];
                unpack16(*reinterpret_cast<const uint4 *>(VsRaw + r * W + vc * VE), f, T());
                float4 *d = reinterpret_cast<float4 *>(Vs + r * W64 + vc * VE);
#pragma unroll
                for (int e = 0; e < VE / 4; ++e) d[e] = make_float4(f[4 * e], f[4 * e + 1], f[4 * e + 2], f[4 * e + 3]);
            }
            if (threadIdx.x < 32) sc[threadIdx.x] = (i0 + threadIdx.x < iend) ? sq[i0 + threadIdx.x] : 0.f;
            __syncthreads();
            if (i0 + 32 < iend) issue(i0 + 32);
        } else {
            stage_rows<T>(Ks, KP, Kp + (row0 + i0) * k_ld + k_off, k_ld, 32, iend - i0, KD, KD4, false);
            stage_rows<T>(Vs, W64, Vp + (row0 + i0) * v_ld + v_off, v_ld, 32, iend - i0, W, W64, false);
            if (threadIdx.x < 32) sc[threadIdx.x] = (i0 + threadIdx.x < iend) ? sq[i0 + threadIdx.x] : 0.f;
            __syncthreads();
        }
        {
            float dot[2][4];
#pragma unroll
            for (int p = 0; p < 2; ++p)
#pragma unroll
                for (int q = 0; q < 4; ++q) dot[p][q] = 0.f;
            const float *ra_p = Rs + rg * KP, *rb_p = Rs + (rg + 32) * KP;
            for (int k = 0; k < KD4; k += 4) {
                const float4 ra = *reinterpret_cast<const float4 *>(ra_p + k);
                const float4 rb = *reinterpret_cast<const float4 *>(rb_p + k);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 kv = *reinterpret_cast<const float4 *>(Ks + (cg + 8 * q) * KP + k);
                    float d0 = dot[0][q], d1 = dot[1][q];
                    d0 = fmaf(ra.x, kv.x, d0);
                    d1 = fmaf(rb.x, kv.x, d1);
                    d0 = fmaf(ra.y, kv.y, d0);
                    d1 = fmaf(rb.y, kv.y, d1);
                    d0 = fmaf(ra.z, kv.z, d0);
                    d1 = fmaf(rb.z, kv.z, d1);
                    d0 = fmaf(ra.w, kv.w, d0);
                    d1 = fmaf(rb.w, kv.w, d1);
                    dot[0][q] = d0;
                    dot[1][q] = d1;
                }
            }
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const int jj = rg + 32 * p, j = j0 + jj;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int ii = cg + 8 * q, i = i0 + ii;
                    const bool ok = jj < jn && i < iend && (kAnti ? i >= j : i <= j);
                    Ms[jj * kMsLd + ii] = ok ? expf(kAnti ? sc[ii] - sr[jj] : sr[jj] - sc[ii]) * dot[p][q] : 0.f;
                }
            }
        }
        __syncthreads();
        for (int ii = 0; ii < 32; ii += 4) {
            float4 mv[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) mv[r] = *reinterpret_cast<const float4 *>(Ms + (ty + 16 * r) * kMsLd + ii);
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
#pragma unroll
                for (int v = 0; v < RV; ++v) {
                    const float4 vv = *reinterpret_cast<const float4 *>(Vs + (ii + e2) * W64 + 64 * v + 4 * tx);
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const float m = e2 == 0 ? mv[r].x : e2 == 1 ? mv[r].y : e2 == 2 ? mv[r].z : mv[r].w;
                        acc[r][v][0] = fmaf(m, vv.x, acc[r][v][0]);
                        acc[r][v][1] = fmaf(m, vv.y, acc[r][v][1]);
                        acc[r][v][2] = fmaf(m, vv.z, acc[r][v][2]);
                        acc[r][v][3] = fmaf(m, vv.w, acc[r][v][3]);
                    }
                }
            }
        }
        __syncthreads();
    }

    const float Dh = a.D ? a.D[h] : 0.f;
    TO *out = static_cast<TO *>(a.out);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int jj = ty + 16 * r;
        if (jj >= jn) continue;
        const size_t tok = row0 + j0 + jj;
        TO *orow = out + (tok * sh.H + h) * W;
#pragma unroll
        for (int v = 0; v < RV; ++v) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int w = 64 * v + 4 * tx + e;
                if (w >= W) continue;
                float val = acc[r][v][e];
                if (a.D) val = fmaf(Dh, to_f32(Vp[tok * v_ld + v_off + w]), val);
                orow[w] = from_f32<TO>(val);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Sum over each group's heads: dB = sum_h dB^(h), dC = sum_h dC^(h) (in the
// input dtype), and each head's dsigma_t = C_t . dC^(h)_t - B_t . dB^(h)_t.
// One warp per (batch, token, group); lanes stride the N columns; heads in
// ascending order.  256 threads per block.
// ---------------------------------------------------------------------------
constexpr int kMaxNPerLane = kMaxN / 32;

template <typename T>
__global__ void __launch_bounds__(256) group_reduce_kernel(const float *__restrict__ dBh, const float *__restrict__ dCh,
                                                           const T *__restrict__ Bm, const T *__restrict__ Cm,
                                                           T *__restrict__ dB, T *__restrict__ dC,
                                                           float *__restrict__ dsig, Shape sh) {
    const long long unit = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const long long units = (long long)sh.batch * sh.T * sh.G;
    if (unit >= units) return;
    const int lane = threadIdx.x & 31;
    const int g = (int)(unit % sh.G);
    const long long tok = unit / sh.G;  // b * T + t
    const int b = (int)(tok / sh.T), t = (int)(tok - (long long)b * sh.T);
    const size_t grow = (size_t)unit * sh.N;  // row (b, t, g) of B, C, dB, dC
    float bv[kMaxNPerLane], cv[kMaxNPerLane], sb[kMaxNPerLane], sc[kMaxNPerLane];
#pragma unroll
    for (int m = 0; m < kMaxNPerLane; ++m) {
        const int n = lane + 32 * m;
        const bool ok = n < sh.N;
        bv[m] = ok ? to_f32(Bm[grow + n]) : 0.f;
        cv[m] = ok ? to_f32(Cm[grow + n]) : 0.f;
        sb[m] = 0.f;
        sc[m] = 0.f;
    }
    // four heads' rows in flight at once; the sums still run in head order
#pragma unroll 4
    for (int hh = 0; hh < sh.heads_per_group; ++hh) {
        const int h = g * sh.heads_per_group + hh;
        const size_t hrow = ((size_t)tok * sh.H + h) * sh.N;
        float d = 0.f;
#pragma unroll
        for (int m = 0; m < kMaxNPerLane; ++m) {
            const int n = lane + 32 * m;
            if (n < sh.N) {
                const float db = dBh[hrow + n], dc = dCh[hrow + n];
                sb[m] += db;
                sc[m] += dc;
                d = fmaf(cv[m], dc, d);
                d = fmaf(-bv[m], db, d);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        if (lane == 0) dsig[((size_t)b * sh.H + h) * sh.T + t] = d;
    }
#pragma unroll
    for (int m = 0; m < kMaxNPerLane; ++m) {
        const int n = lane + 32 * m;
        if (n < sh.N) {
            dB[grow + n] = from_f32<T>(sb[m]);
            dC[grow + n] = from_f32<T>(sc[m]);
        }
    }
}

// The same sums with each lane on 4 consecutive n (16-byte loads of the per-head terms, 8 or 16 bytes of
// B, C, dB, dC), for N a multiple of 4 and aligned rows: a row of 128 is one load per lane, and eight
// heads' rows (four for N above 128) are in flight at once; the sums over heads still run in head order.
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    const uint2 r = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&r.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&r.y);
    return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
}
__device__ __forceinline__ void store4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16 *p, float4 v) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 r;
    r.x = *reinterpret_cast<const uint32_t *>(&a);
    r.y = *reinterpret_cast<const uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = r;
}

// kNV: 4-vectors per lane (1 for N up to 128, 2 up to 256)
template <typename T, int kNV>
__global__ void __launch_bounds__(256) group_reduce_vec_kernel(const float *__restrict__ dBh,
                                                               const float *__restrict__ dCh,
                                                               const T *__restrict__ Bm, const T *__restrict__ Cm,
                                                               T *__restrict__ dB, T *__restrict__ dC,
                                                               float *__restrict__ dsig, Shape sh) {
    const long long unit = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const long long units = (long long)sh.batch * sh.T * sh.G;
    if (unit >= units) return;
    const int lane = threadIdx.x & 31;
    const int g = (int)(unit % sh.G);
    const long long tok = unit / sh.G;  // b * T + t
    const int b = (int)(tok / sh.T), t = (int)(tok - (long long)b * sh.T);
    const size_t grow = (size_t)unit * sh.N;  // row (b, t, g) of B, C, dB, dC
    const int V = sh.N / 4;                   // 4-vectors per row
    float4 bv[kNV], cv[kNV], sb[kNV], sc[kNV];
#pragma unroll
    for (int m = 0; m < kNV; ++m) {
        const int v = lane + 32 * m;
        const bool ok = v < V;
        bv[m] = ok ? load4(Bm + grow + 4 * v) : make_float4(0.f, 0.f, 0.f, 0.f);
        cv[m] = ok ? load4(Cm + grow + 4 * v) : make_float4(0.f, 0.f, 0.f, 0.f);
        sb[m] = make_float4(0.f, 0.f, 0.f, 0.f);
        sc[m] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll(8 / kNV)
    for (int hh = 0; hh < sh.heads_per_group; ++hh) {
        const int h = g * sh.heads_per_group + hh;
        const size_t hrow = ((size_t)tok * sh.H + h) * sh.N;
        float d = 0.f;
#pragma unroll
        for (int m = 0; m < kNV; ++m) {
            const int v = lane + 32 * m;
            if (v < V) {
                const float4 db = load4(dBh + hrow + 4 * v), dc = load4(dCh + hrow + 4 * v);
                sb[m].x += db.x; sb[m].y += db.y; sb[m].z += db.z; sb[m].w += db.w;
                sc[m].x += dc.x; sc[m].y += dc.y; sc[m].z += dc.z; sc[m].w += dc.w;
                d = fmaf(cv[m].x, dc.x, d);
                d = fmaf(-bv[m].x, db.x, d);
                d = fmaf(cv[m].y, dc.y, d);
                d = fmaf(-bv[m].y, db.y, d);
                d = fmaf(cv[m].z, dc.z, d);
                d = fmaf(-bv[m].z, db.z, d);
                d = fmaf(cv[m].w, dc.w, d);
                d = fmaf(-bv[m].w, db.w, d);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        if (lane == 0) dsig[((size_t)b * sh.H + h) * sh.T + t] = d;
    }
#pragma unroll
    for (int m = 0; m < kNV; ++m) {
        const int v = lane + 32 * m;
        if (v < V) {
            store4(dB + grow + 4 * v, sb[m]);
            store4(dC + grow + 4 * v, sc[m]);
        }
    }
}

// ---------------------------------------------------------------------------
// Per (head, batch): the suffix sums of dsigma over the whole sequence (fp64),
// plus <dfinal, final> at the last token, give d(dt_u A_h); write
// ddt = A_h d(dt A), and the batch row's shares of dA = sum dt d(dt A) and
// dD = sum <dy, x> (fp64).  grid (H, batch, kDdSlices), 256 threads: slice 0
// runs the suffix sums (each thread owns a contiguous run of tokens, a block
// scan of the run totals gives each run the sum of the runs after it); every
// slice sums dD over its quarter of the tokens.
// ---------------------------------------------------------------------------
constexpr int kDtThreads = 256;

__device__ double block_sum(double v, double *red) {
    red[threadIdx.x] = v;
    __syncthreads();
    for (int o = kDtThreads / 2; o > 0; o >>= 1) {
        if ((int)threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    const double r = red[0];
    __syncthreads();
    return r;
}

template <typename T>
__global__ void __launch_bounds__(kDtThreads) dt_scan_kernel(const float *__restrict__ dsig,
                                                             const float *__restrict__ dt,
                                                             const float *__restrict__ A, const T *__restrict__ x,
                                                             const T *__restrict__ dy,
                                                             const float *__restrict__ dfin,
                                                             const float *__restrict__ fin, float *__restrict__ ddt,
                                                             double *__restrict__ pa, double *__restrict__ pd,
                                                             Shape sh, int vec) {
    __shared__ double red[kDtThreads];
    __shared__ double suf[kDtThreads];
    const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, z = blockIdx.z;
    const size_t bh = (size_t)b * sh.H + h;
    const size_t PN = (size_t)sh.P * sh.N;
    // the tokens of this block's dD slice
    const int tq = (sh.T + kDdSlices - 1) / kDdSlices, tlo = min(sh.T, z * tq), thi = min(sh.T, tlo + tq);
    if (z == 0) {
        double fd = 0.0;
        if (dfin)
            for (size_t e = tid; e < PN; e += kDtThreads) fd += (double)dfin[bh * PN + e] * (double)fin[bh * PN + e];
        const double fdot = block_sum(fd, red);

        const float *ds = dsig + bh * sh.T;
        const int run = (sh.T + kDtThreads - 1) / kDtThreads;
        const int t0 = min(sh.T, tid * run), t1 = min(sh.T, t0 + run);
        double part = 0.0;
        for (int t = t0; t < t1; ++t) part += (double)ds[t];
        suf[tid] = part;
        __syncthreads();
        // inclusive suffix scan of the run totals
        for (int o = 1; o < kDtThreads; o <<= 1) {
            const double v = tid + o < kDtThreads ? suf[tid + o] : 0.0;
            __syncthreads();
            suf[tid] += v;
            __syncthreads();
    }
    double acc = (tid + 1 < kDtThreads ? suf[tid + 1] : 0.0) + fdot;
    const double Ah = (double)A[h];
    double da = 0.0;
    for (int t = t1 - 1; t >= t0; --t) {
        acc += (double)ds[t];
        const size_t it = ((size_t)b * sh.T + t) * sh.H + h;
        ddt[it] = (float)(Ah * acc);
        da += (double)dt[it] * acc;
    }
    const double dA_part = block_sum(da, red);
    if (tid == 0) pa[bh] = dA_part;
    }

    // dD's share: sum over the row's tokens of <dy_t, x_t> for this head.  With 16-byte rows, eight
    // elements per load (their products summed in fp32, then in fp64), four loads in flight per thread.
    double dd = 0.0;
    constexpr int VE = 16 / (int)sizeof(T);
    if (vec) {
        const int cpt = sh.P / VE;  // 16-byte pieces per token row
        const long long total = (long long)thi * cpt;
#pragma unroll 4
        for (long long idx = (long long)tlo * cpt + tid; idx < total; idx += kDtThreads) {
            const int t = (int)(idx / cpt), q = (int)(idx - (long long)t * cpt);
            const size_t off = (((size_t)b * sh.T + t) * sh.H + h) * sh.P + (size_t)q * VE;
            float fy[VE], fx[VE];
            unpack16(*reinterpret_cast<const uint4 *>(dy + off), fy, T());
            unpack16(*reinterpret_cast<const uint4 *>(x + off), fx, T());
            float f = 0.f;
#pragma unroll
            for (int e = 0; e < VE; ++e) f = fmaf(fy[e], fx[e], f);
            dd += (double)f;
        }
    } else {
        const long long TP = (long long)thi * sh.P;
        for (long long idx = (long long)tlo * sh.P + tid; idx < TP; idx += kDtThreads) {
            const int t = (int)(idx / sh.P), p = (int)(idx - (long long)t * sh.P);
            const size_t off = (((size_t)b * sh.T + t) * sh.H + h) * sh.P + p;
            dd += (double)to_f32(dy[off]) * (double)to_f32(x[off]);
        }
    }
    const double dD_part = block_sum(dd, red);
    if (tid == 0) pd[(size_t)z * sh.batch * sh.H + bh] = dD_part;
}

// dA[h] = sum_b pa[b][h], dD[h] = sum_b sum_z pd[z][b][h], in batch order (and slice order).
__global__ void __launch_bounds__(256) param_reduce_kernel(const double *__restrict__ pa,
                                                           const double *__restrict__ pd, float *__restrict__ dA,
                                                           float *__restrict__ dD, int batch, int H) {
    const int h = blockIdx.x * 256 + threadIdx.x;
    if (h >= H) return;
    double sa = 0.0, sd = 0.0;
    for (int b = 0; b < batch; ++b) {
        sa += pa[(size_t)b * H + h];
        for (int z = 0; z < kDdSlices; ++z) sd += pd[((size_t)z * batch + b) * H + h];
    }
    dA[h] = (float)sa;
    dD[h] = (float)sd;
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
size_t scan_smem_bytes(int KD, int W, size_t es, bool vec) {
    const size_t KP = (size_t)((KD + 3) & ~3) + 4, W64 = (size_t)64 * ((W + 63) / 64);
    const size_t raw = vec ? 32 * (size_t)(KD + W) * es : 0;
    return sizeof(float) * (96 * KP + 32 * W64 + 32 * (W64 + 4) + 64 * kMsLd + 96 + kMaxQ) + raw;
}

template <typename T, typename TO, int RV, bool kAnti>
cudaError_t launch_scan_rv(const ScanArgs &a, const float *s, const Shape &sh, cudaStream_t st) {
    const size_t smem = scan_smem_bytes(a.KD, a.W, sizeof(T), a.vec != 0);
    auto k = masked_scan_kernel<T, TO, RV, kAnti>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int tiles = (sh.Q + 63) / 64;
    k<<<dim3(sh.nc * tiles, sh.H, sh.batch), 256, smem, st>>>(a, s, sh);
    return cudaGetLastError();
}

template <typename T, typename TO, bool kAnti>
cudaError_t launch_scan(const ScanArgs &a, const float *s, const Shape &sh, cudaStream_t st) {
    switch ((a.W + 63) / 64) {
        case 1: return launch_scan_rv<T, TO, 1, kAnti>(a, s, sh, st);
        case 2: return launch_scan_rv<T, TO, 2, kAnti>(a, s, sh, st);
        case 3: return launch_scan_rv<T, TO, 3, kAnti>(a, s, sh, st);
        default: return launch_scan_rv<T, TO, 4, kAnti>(a, s, sh, st);
    }
}

bool is_aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool ranges_overlap(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || !na || !nb) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// dt, A and D gradients from dsigma: the dt scan, then the parameter sums
template <typename T>
int run_dt_tail(const Shape &sh, const float *dsig, const float *dt, const float *A, const T *x, const T *dy,
                const float *dfin, const float *fin, float *ddt, float *dA, float *dD, double *pa, double *pd, int vec,
                cudaStream_t st) {
    dt_scan_kernel<T><<<dim3(sh.H, sh.batch, kDdSlices), kDtThreads, 0, st>>>(dsig, dt, A, x, dy, dfin, fin, ddt, pa,
                                                                           pd, sh, vec);
    if (cudaGetLastError() != cudaSuccess) return SSD_ERR_CUDA;
    param_reduce_kernel<<<(sh.H + 255) / 256, 256, 0, st>>>(pa, pd, dA, dD, sh.batch, sh.H);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

template <typename T>
int run_bwd(const Shape &sh, const T *x, const float *dt, const float *A, const T *B, const T *C, const float *D,
            const float *init, const T *dy, const float *dfin, T *dx, float *ddt, float *dA, T *dB, T *dC,
            float *dD, float *dinit, char *ws, const BwdWorkspace &w, cudaStream_t st) {
    float *s = reinterpret_cast<float *>(ws + w.s_off);
    float *Hin = reinterpret_cast<float *>(ws + w.hin_off);
    float *Gout = reinterpret_cast<float *>(ws + w.gout_off);
    float *fin = reinterpret_cast<float *>(ws + w.fin_off);
    float *dBh = reinterpret_cast<float *>(ws + w.dbh_off);
    float *dCh = reinterpret_cast<float *>(ws + w.dch_off);
    float *dsig = reinterpret_cast<float *>(ws + w.dsig_off);
    double *pa = reinterpret_cast<double *>(ws + w.pa_off);
    double *pd = reinterpret_cast<double *>(ws + w.pd_off);
    int *status = reinterpret_cast<int *>(ws + w.status_off);
    if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return SSD_ERR_CUDA;
    if (launch_chunk_cumsum(dt, A, s, sh, st) != cudaSuccess) return SSD_ERR_CUDA;
    // 16-byte operand loads need 16-byte aligned tensors whose rows are whole vectors
    constexpr int VE = 16 / (int)sizeof(T);
    const bool al = is_aligned(x, 16) && is_aligned(dy, 16) && is_aligned(B, 16) && is_aligned(C, 16);
    const bool cs_tc = chunk_state_tc_supported(sh, sizeof(T) == 2 ? SSD_BF16 : SSD_F32) && al;
    auto chunk_states = [&](const T *xx, const T *bb, float *out, bool from_start) {
        return cs_tc ? launch_chunk_state_tc(xx, bb, s, out, from_start, status, sh, st)
                     : launch_chunk_state<T>(xx, bb, s, out, sh, st, from_start);
    };
    // forward states: Hin_c, and the final state when a final-state gradient is given
    if (chunk_states(x, B, Hin, false) != cudaSuccess) return SSD_ERR_CUDA;
    if (launch_state_passing(Hin, s, init, dfin ? fin : nullptr, sh, st) != cudaSuccess) return SSD_ERR_CUDA;
    // backward states: sum_i exp(s_i) dy_i C_i^T per chunk, then dHout_c and dinit
    if (chunk_states(dy, C, Gout, true) != cudaSuccess) return SSD_ERR_CUDA;
    const int PN = sh.P * sh.N;
    if (PN % 4 == 0 && reinterpret_cast<uintptr_t>(dfin) % 16 == 0 && reinterpret_cast<uintptr_t>(dinit) % 16 == 0)
        state_passing_bwd_vec_kernel<<<dim3((PN + 1023) / 1024, sh.H, sh.batch), 256, 0, st>>>(Gout, s, dfin, dinit,
                                                                                             sh);
    else
        state_passing_bwd_kernel<<<dim3((PN + 255) / 256, sh.H, sh.batch), 256, 0, st>>>(Gout, s, dfin, dinit, sh);
    if (cudaGetLastError() != cudaSuccess) return SSD_ERR_CUDA;
    const int vec = al && sh.P % VE == 0 && sh.N % VE == 0;
    const int st_vec = sh.P % 4 == 0 && sh.N % 4 == 0;
    // The three masked scans: on the tensor cores (ssd_bwd_tc.cu) for bf16 inputs with P = 64, N in {64, 128},
    // Q in {128, 256} and 16-byte aligned tensors, else on the CUDA cores.
    const bool tc = scan_tc_supported(sh, sizeof(T) == 2 ? SSD_BF16 : SSD_F32) && al && kScanTcRoles != 0;
    // dx: rows of B against columns of C, values dy, state dHout as [P][N] = [W][KD], skip D dy
    if (tc && (kScanTcRoles & 1)) {
        if (launch_masked_scan_tc(B, 0, C, 0, dy, 1, sh.N, sh.P, true, Gout, 0, D, dx, true, s, status, sh, st) !=
            cudaSuccess)
            return SSD_ERR_CUDA;
    } else {
        ScanArgs ax{B, C, dy, 0, 0, 1, Gout, 0, sh.N, sh.P, D, dx, vec, st_vec};
        if (launch_scan<T, T, true>(ax, s, sh, st) != cudaSuccess) return SSD_ERR_CUDA;
    }
    // dB and dC summed over each group's heads inside the scans (their per-head terms never reach memory):
    // the dot products with B and C rows that dsigma needs are taken there too
    if (tc && (kScanTcRoles & 6) == 6 && sh.Q % 128 == 0) {
        float *partB = dBh, *partC = dCh;
        float *dotB = reinterpret_cast<float *>(ws + w.dbh_off + bwd_sum_dot_off(sh));
        float *dotC = reinterpret_cast<float *>(ws + w.dch_off + bwd_sum_dot_off(sh));
        if (launch_masked_scan_tc(x, 1, dy, 1, C, 0, sh.P, sh.N, true, Gout, 1, nullptr, nullptr, false, s, status, sh,
                                  st, B, dotB, partB) != cudaSuccess ||
            launch_masked_scan_tc(dy, 1, x, 1, B, 0, sh.P, sh.N, false, Hin, 1, nullptr, nullptr, false, s, status,
                                  sh, st, C, dotC, partC) != cudaSuccess ||
            launch_head_sum_reduce(partB, dotB, partC, dotC, dB, dC, dsig, sh, st) != cudaSuccess)
            return SSD_ERR_CUDA;
        return run_dt_tail(sh, dsig, dt, A, x, dy, dfin, fin, ddt, dA, dD, pa, pd, vec, st);
    }
    // dB^(h): rows of x against columns of dy, values C, state dHout as [P][N] = [KD][W]
    if (tc && (kScanTcRoles & 2)) {
        if (launch_masked_scan_tc(x, 1, dy, 1, C, 0, sh.P, sh.N, true, Gout, 1, nullptr, dBh, false, s, status, sh,
                                  st) != cudaSuccess)
            return SSD_ERR_CUDA;
    } else {
        ScanArgs ab{x, dy, C, 1, 1, 0, Gout, 1, sh.P, sh.N, nullptr, dBh, vec, st_vec};
        if (launch_scan<T, float, true>(ab, s, sh, st) != cudaSuccess) return SSD_ERR_CUDA;
    }
    // dC^(h): rows of dy against columns of x, values B, state Hin as [P][N] = [KD][W]
    if (tc && (kScanTcRoles & 4)) {
        if (launch_masked_scan_tc(dy, 1, x, 1, B, 0, sh.P, sh.N, false, Hin, 1, nullptr, dCh, false, s, status, sh,
                                  st) != cudaSuccess)
            return SSD_ERR_CUDA;
    } else {
        ScanArgs ac{dy, x, B, 1, 1, 0, Hin, 1, sh.P, sh.N, nullptr, dCh, vec, st_vec};
        if (launch_scan<T, float, false>(ac, s, sh, st) != cudaSuccess) return SSD_ERR_CUDA;
    }
    const long long units = (long long)sh.batch * sh.T * sh.G;
    // the vector form wants rows of B, C, dB, dC aligned to their 4-vectors (N a multiple of 4)
    const size_t a4 = 4 * sizeof(T);
    const bool gvec = sh.N % 4 == 0 && reinterpret_cast<uintptr_t>(B) % a4 == 0 &&
                      reinterpret_cast<uintptr_t>(C) % a4 == 0 && reinterpret_cast<uintptr_t>(dB) % a4 == 0 &&
                      reinterpret_cast<uintptr_t>(dC) % a4 == 0;
    if (gvec && sh.N <= 128)
        group_reduce_vec_kernel<T, 1><<<(unsigned)((units + 7) / 8), 256, 0, st>>>(dBh, dCh, B, C, dB, dC, dsig, sh);
    else if (gvec)
        group_reduce_vec_kernel<T, 2><<<(unsigned)((units + 7) / 8), 256, 0, st>>>(dBh, dCh, B, C, dB, dC, dsig, sh);
    else
        group_reduce_kernel<T><<<(unsigned)((units + 7) / 8), 256, 0, st>>>(dBh, dCh, B, C, dB, dC, dsig, sh);
    if (cudaGetLastError() != cudaSuccess) return SSD_ERR_CUDA;
    return run_dt_tail(sh, dsig, dt, A, x, dy, dfin, fin, ddt, dA, dD, pa, pd, vec, st);
}

}  // namespace
}  // namespace ssd

extern "C" int ssd_bwd_check(const void *workspace, void *stream) {
    if (!workspace) return SSD_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return SSD_ERR_CUDA;
    int status = 0;  // the status word heads the backward's workspace
    if (cudaMemcpy(&status, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SSD_ERR_CUDA;
    return status;
}

extern "C" size_t ssd_bwd_workspace_bytes(int batch, int T, int H, int P, int G, int N, int Q, int dtype) {
    ssd::Shape sh;
    if (ssd::check_dims(batch, T, H, P, G, N, Q, dtype, &sh) != SSD_OK) return 0;
    return ssd::bwd_layout(sh).total;
}

extern "C" int ssd_bwd(const void *x, const float *dt, const float *A, const void *B, const void *C, const float *D,
                       int Q, const float *init_state, const void *dy, const float *dfinal_state, void *dx,
                       float *ddt, float *dA, void *dB, void *dC, float *dD, float *dinit_state, int batch, int T,
                       int H, int P, int G, int N, int dtype, void *workspace, size_t workspace_bytes,
                       void *stream) {
    ssd::Shape sh;
    int rc = ssd::check_dims(batch, T, H, P, G, N, Q, dtype, &sh);
    if (rc != SSD_OK) return rc;
    if ((T > 0 && (!x || !dt || !B || !C || !dy || !dx || !ddt || !dB || !dC)) || !A || !D || !dA || !dD ||
        !workspace)
        return SSD_ERR_INVALID_ARG;
    if (batch > 65535 || H > 65535) return SSD_ERR_UNSUPPORTED;
    const size_t es = (dtype == SSD_BF16) ? 2 : 4;
    using ssd::is_aligned;
    if (!is_aligned(x, es) || !is_aligned(B, es) || !is_aligned(C, es) || !is_aligned(dy, es) ||
        !is_aligned(dx, es) || !is_aligned(dB, es) || !is_aligned(dC, es) || !is_aligned(dt, 4) ||
        !is_aligned(A, 4) || !is_aligned(D, 4) || !is_aligned(ddt, 4) || !is_aligned(dA, 4) || !is_aligned(dD, 4) ||
        !is_aligned(init_state, 4) || !is_aligned(dfinal_state, 4) || !is_aligned(dinit_state, 4) ||
        !is_aligned(workspace, 256))
        return SSD_ERR_INVALID_ARG;
    const ssd::BwdWorkspace w = ssd::bwd_layout(sh);
    if (workspace_bytes < w.total) return SSD_ERR_INVALID_ARG;
    // outputs may not overlap any input or one another
    const size_t xb = es * (size_t)batch * T * H * P, bcb = es * (size_t)batch * T * G * N;
    const size_t tb = sizeof(float) * (size_t)batch * T * H, hb = sizeof(float) * H;
    const size_t sb = sizeof(float) * (size_t)batch * H * P * N;
    const void *ins[] = {x, dt, A, B, C, D, init_state, dy, dfinal_state};
    const size_t insz[] = {xb, tb, hb, bcb, bcb, hb, sb, xb, sb};
    const void *outs[] = {dx, ddt, dA, dB, dC, dD, dinit_state, workspace};
    const size_t outsz[] = {xb, tb, hb, bcb, bcb, hb, sb, w.total};
    for (int i = 0; i < 8; ++i) {
        for (int j = 0; j < 9; ++j)
            if (ssd::ranges_overlap(outs[i], outsz[i], ins[j], insz[j])) return SSD_ERR_INVALID_ARG;
        for (int j = i + 1; j < 8; ++j)
            if (ssd::ranges_overlap(outs[i], outsz[i], outs[j], outsz[j])) return SSD_ERR_INVALID_ARG;
    }

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) {
        // final = init: the gradient passes straight through; nothing else depends on the inputs
        if (cudaMemsetAsync(dA, 0, hb, st) != cudaSuccess || cudaMemsetAsync(dD, 0, hb, st) != cudaSuccess)
            return SSD_ERR_CUDA;
        if (!dinit_state) return SSD_OK;
        cudaError_t e = dfinal_state
                            ? cudaMemcpyAsync(dinit_state, dfinal_state, sb, cudaMemcpyDeviceToDevice, st)
                            : cudaMemsetAsync(dinit_state, 0, sb, st);
        return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
    }
    char *ws = static_cast<char *>(workspace);
    if (dtype == SSD_BF16) {
        using bf = __nv_bfloat16;
        return ssd::run_bwd<bf>(sh, static_cast<const bf *>(x), dt, A, static_cast<const bf *>(B),
                                static_cast<const bf *>(C), D, init_state, static_cast<const bf *>(dy),
                                dfinal_state, static_cast<bf *>(dx), ddt, dA, static_cast<bf *>(dB),
                                static_cast<bf *>(dC), dD, dinit_state, ws, w, st);
    }
    return ssd::run_bwd<float>(sh, static_cast<const float *>(x), dt, A, static_cast<const float *>(B),
                               static_cast<const float *>(C), D, init_state, static_cast<const float *>(dy),
                               dfinal_state, static_cast<float *>(dx), ddt, dA, static_cast<float *>(dB),
                               static_cast<float *>(dC), dD, dinit_state, ws, w, st);
}
