// ssd_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) chunk scan of the SSD
// forward for bf16 inputs: stages 1, 4 and 5 of the block decomposition of
// "Transformers are SSMs" (analysis page, section "The Block-Decomposition SSD
// Algorithm") plus the D skip, for one 128-row half of a chunk and a block of
// heads that share one B/C group:
//
//   G   = C_r B^T                         (C rows of this half, B rows 0..end of half)
//   Y   = exp(s_j) * (C_r S~_{c-1}^T)     (stage 4: inter-chunk output)
//   M   = G o exp(s_j - s_i) [i <= j],  M[j][j] += D_h
//   Y  += M X                             (stage 1 + skip: the masked quadratic form)
//   y   = bf16(Y)                         (stage 5)
//
// G is computed once per unit on the tensor cores into TMEM (fp32) and shared
// by the unit's heads; every head's mask M is built from it by the CUDA cores
// straight into TMEM as the bf16 A operand of the X product.
//
// Decays are always exponentials of non-positive differences: below the
// diagonal 32x32 blocks, exp(s_j - s_i) = exp(s_j - s_k) * exp(s_k - s_i)
// with s_k the last column of the 32-column slab (one exponential per row per
// slab, one per column per head); inside a diagonal block the exponential is
// taken per element.
#include "ssd_common.cuh"
#include "tc_prims.cuh"
#include "tma_host.h"

namespace ssd {

using namespace tc;

namespace {

constexpr int kThreads = 256;  // two warpgroups; each covers the 128 TMEM lanes
constexpr int kRows = 128;     // rows of a chunk half (the UMMA M)
constexpr int kP = 64;         // head dimension supported by this path

// TMEM columns (fp32 words): G [0, 256), M (bf16 pairs) [256, 384), Y [384, 448).
constexpr uint32_t kColG = 0, kColM = 256, kColY = 384, kTmemCols = 512;

// Shared memory carve-up (bytes from a 1 KiB-aligned base).
constexpr uint32_t kOffC = 0;                  // 2 K-atoms x 128 rows x 128 B
constexpr uint32_t kOffB = kOffC + 2 * 16384;  // 2 K-atoms x 256 rows x 128 B
constexpr uint32_t kOffX = kOffB + 2 * 32768;  // 256 rows x 128 B (MN-major)
constexpr uint32_t kOffS = kOffX + 32768;      // 2 K-atoms x 64 rows x 128 B
constexpr uint32_t kOffJ = kOffS + 2 * 8192;   // float s[256]
constexpr uint32_t kOffF = kOffJ + 1024;       // float column factors[256]
constexpr uint32_t kSmemBytes = kOffF + 1024 + 1024;  // + alignment slack

struct ScanParams {
    Shape sh;
    const float *s;      // [b][H][nc][Q]
    const float *Sprev;  // [b][nc][H][P][N]: state entering each chunk
    const float *D;      // [H]
    __nv_bfloat16 *y;    // [b][T][H][P]
    int *status;
    int NK;              // K-atoms of 64 along N
    int halves;          // Q / 128
    int heads_per_unit;
    int blocks_per_group;
    int n_units;
};

__device__ __forceinline__ uint8_t *align_1k(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    chunk_scan_tc_kernel(const __grid_constant__ CUtensorMap mC, const __grid_constant__ CUtensorMap mB,
                         const __grid_constant__ CUtensorMap mX, const ScanParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint8_t *sC = smem + kOffC;
    uint8_t *sB = smem + kOffB;
    uint8_t *sX = smem + kOffX;
    uint8_t *sS = smem + kOffS;
    float *sJ = reinterpret_cast<float *>(smem + kOffJ);
    float *sF = reinterpret_cast<float *>(smem + kOffF);
    __shared__ uint64_t bar_cb, bar_x, bar_mma;
    __shared__ uint32_t tslot;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int wg = warp >> 2;                 // warpgroup 0 or 1
    const int row = ((warp & 3) << 5) + lane; // TMEM lane = row within the half
    const Shape sh = p.sh;
    const int N = sh.N, NK = p.NK;

    if (warp == 0) tmem_alloc(&tslot, kTmemCols);
    if (tid == 0) {
        mbar_init(&bar_cb, 1);
        mbar_init(&bar_x, 1);
        mbar_init(&bar_mma, 1);
        mbar_fence_init();
        tma_prefetch_desc(&mC);
        tma_prefetch_desc(&mB);
        tma_prefetch_desc(&mX);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    const uint32_t tG = tmem + kColG, tM = tmem + kColM, tY = tmem + kColY;
    const uint32_t lane_base = (uint32_t)((warp & 3) << 5) << 16;  // this warp's TMEM lane quadrant
    uint32_t ph_cb = 0, ph_x = 0, ph_mma = 0;
    // A bounded wait that gives up sets `fail`; barriers OR it across the CTA so
    // every thread leaves the loops together (the status word is already set).
    int fail = 0;
    bool aborted = false;

    for (int u = blockIdx.x; u < p.n_units && !aborted; u += gridDim.x) {
        // unit -> (b, c, half r, group g, head block)
        int rem = u;
        const int hb = rem % p.blocks_per_group;
        rem /= p.blocks_per_group;
        const int g = rem % sh.G;
        rem /= sh.G;
        const int r = rem % p.halves;
        rem /= p.halves;
        const int c = rem % sh.nc;
        const int b = rem / sh.nc;
        const int h_first = g * sh.heads_per_group + hb * p.heads_per_unit;
        const int h_last = min(h_first + p.heads_per_unit, (g + 1) * sh.heads_per_group);
        const int t0 = c * sh.Q;
        const int len = min(sh.Q, sh.T - t0);
        const int row0 = r * kRows;
        if (row0 >= len) continue;  // this half lies past the end of the sequence
        const int kcols = row0 + kRows;  // columns i of the masked product: [0, kcols)
        const int nbox = kcols / kRows;

        // C rows of this half and B rows [0, kcols), K-major, 128-byte swizzle
        if (tid == 0) {
            mbar_arrive_expect_tx(&bar_cb, (uint32_t)NK * 16384u * (1 + nbox));
            for (int k = 0; k < NK; ++k) {
                tma_load_4d(sC + k * 16384, &mC, &bar_cb, k * 64, g, t0 + row0, b);
                for (int q = 0; q < nbox; ++q)
                    tma_load_4d(sB + k * 32768 + q * 16384, &mB, &bar_cb, k * 64, g, t0 + q * kRows, b);
            }
        }
        fail |= !mbar_wait(&bar_cb, ph_cb, p.status);
        ph_cb ^= 1;
        if (__syncthreads_or(fail)) {
            aborted = true;
            break;
        }
        // G = C_r B^T into TMEM (committed together with the first head's inter product)
        if (tid == 0) {
            fence_after_sync();
            const uint32_t id = idesc_bf16_f32(kRows, kcols, 0, 0);
            for (int kk = 0; kk < NK * 4; ++kk) {
                const int atom = kk >> 2, kin = kk & 3;
                const uint64_t ad = smem_desc_sw128(smem_u32(sC) + atom * 16384 + kin * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(smem_u32(sB) + atom * 32768 + kin * 32, 16, 1024);
                mma_ss(tG, ad, bd, id, kk > 0);
            }
        }

        for (int h = h_first; h < h_last && !aborted; ++h) {
            // X rows [0, kcols) of head h (MN-major B operand of the masked product)
            if (tid == 0) {
                mbar_arrive_expect_tx(&bar_x, (uint32_t)nbox * 16384u);
                for (int q = 0; q < nbox; ++q) tma_load_4d(sX + q * 16384, &mX, &bar_x, 0, h, t0 + q * kRows, b);
            }
            // log-decay prefix sums of this head's chunk
            const float *sc = p.s + (((size_t)b * sh.H + h) * sh.nc + c) * sh.Q;
            for (int i = tid; i < kcols; i += kThreads) sJ[i] = sc[i];
            // state entering the chunk, fp32 [P][N] -> bf16 K-major swizzled tile [64 rows p][N]
            {
                const float *Sp = p.Sprev + (((size_t)b * sh.nc + c) * sh.H + h) * (size_t)kP * N;
                const int chunks = kP * NK * 8;  // 16-byte chunks of 8 bf16
                for (int idx = tid; idx < chunks; idx += kThreads) {
                    const int pr = idx / (NK * 8), n = (idx % (NK * 8)) * 8;
                    uint4 v = make_uint4(0, 0, 0, 0);
                    if (n < N) {
                        const float4 a = *reinterpret_cast<const float4 *>(Sp + (size_t)pr * N + n);
                        const float4 bq = *reinterpret_cast<const float4 *>(Sp + (size_t)pr * N + n + 4);
                        v.x = pack_bf16x2(a.x, a.y);
                        v.y = pack_bf16x2(a.z, a.w);
                        v.z = pack_bf16x2(bq.x, bq.y);
                        v.w = pack_bf16x2(bq.z, bq.w);
                    }
                    const int atom = n >> 6, ch = (n & 63) >> 3;
                    *reinterpret_cast<uint4 *>(sS + atom * 8192 + pr * 128 + ((ch ^ (pr & 7)) << 4)) = v;
                }
            }
            fence_view_async_shared();
            __syncthreads();
            // per-column decay to the end of its 32-column slab: exp(s_{i|31} - s_i) <= 1
            for (int i = tid; i < kcols; i += kThreads) sF[i] = expf(sJ[i | 31] - sJ[i]);
            // stage 4 product: Y = C_r S~^T  (K = N)
            if (tid == 0) {
                fence_after_sync();
                const uint32_t id = idesc_bf16_f32(kRows, kP, 0, 0);
                for (int kk = 0; kk < NK * 4; ++kk) {
                    const int atom = kk >> 2, kin = kk & 3;
                    const uint64_t ad = smem_desc_sw128(smem_u32(sC) + atom * 16384 + kin * 32, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(smem_u32(sS) + atom * 8192 + kin * 32, 16, 1024);
                    mma_ss(tY, ad, bd, id, kk > 0);
                }
                mma_commit(&bar_mma);
            }
            fail |= !mbar_wait(&bar_mma, ph_mma, p.status);
            ph_mma ^= 1;
            if (__syncthreads_or(fail)) {  // also makes sF visible
                aborted = true;
                break;
            }
            fence_after_sync();
            const int j = row0 + row;  // this thread's row within the chunk
            const float sj = sJ[j];
            // Y *= exp(s_j): the decay from the chunk start (warpgroup wg takes 32 columns)
            {
                const float e = expf(sj);
                uint32_t v[16];
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const uint32_t ta = tmem_addr(tY, 0, wg * 32 + hf * 16) + lane_base;
                    tmem_ld16(ta, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 16; ++q) v[q] = __float_as_uint(__uint_as_float(v[q]) * e);
                    tmem_st16(ta, v);
                }
            }
            // mask: M[j][i] = G[j][i] * exp(s_j - s_i) for i <= j, + D_h on the diagonal
            const float Dh = p.D[h];
            for (int slab = wg; slab < kcols / 32; slab += 2) {
                const int i0 = slab * 32;
                uint32_t gv[32];
                tmem_ld16(tmem_addr(tG, 0, i0) + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&gv[0]));
                tmem_ld16(tmem_addr(tG, 0, i0 + 16) + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&gv[16]));
                tmem_wait_ld();
                uint32_t o[16];
                if (i0 + 31 < j) {
                    const float rf = expf(sj - sJ[i0 + 31]);
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const float a = __uint_as_float(gv[2 * q]) * (rf * sF[i0 + 2 * q]);
                        const float bb = __uint_as_float(gv[2 * q + 1]) * (rf * sF[i0 + 2 * q + 1]);
                        o[q] = pack_bf16x2(a, bb);
                    }
                } else if (i0 > j) {
#pragma unroll
                    for (int q = 0; q < 16; ++q) o[q] = 0u;
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const int ia = i0 + 2 * q, ib = ia + 1;
                        float a = (ia <= j) ? __uint_as_float(gv[2 * q]) * expf(sj - sJ[ia]) : 0.f;
                        float bb = (ib <= j) ? __uint_as_float(gv[2 * q + 1]) * expf(sj - sJ[ib]) : 0.f;
                        if (ia == j) a += Dh;
                        if (ib == j) bb += Dh;
                        o[q] = pack_bf16x2(a, bb);
                    }
                }
                tmem_st16(tmem_addr(tM, 0, i0 / 2) + lane_base, o);
            }
            tmem_wait_st();
            fence_before_sync();
            if (tid == 0) fail |= !mbar_wait(&bar_x, ph_x, p.status);
            ph_x ^= 1;
            if (__syncthreads_or(fail)) {
                aborted = true;
                break;
            }
            // stage 1 product: Y += M X  (K = kcols)
            if (tid == 0) {
                fence_after_sync();
                const uint32_t id = idesc_bf16_f32(kRows, kP, 0, 1);
                for (int kk = 0; kk < kcols / 16; ++kk) {
                    const uint64_t bd = smem_desc_sw128(smem_u32(sX) + kk * 2048, 16, 1024);
                    mma_ts(tY, tM + kk * 8, bd, id, 1);
                }
                mma_commit(&bar_mma);
            }
            fail |= !mbar_wait(&bar_mma, ph_mma, p.status);
            ph_mma ^= 1;
            fence_after_sync();
            // stage 5: y = bf16(Y) for rows inside the sequence
            {
                uint32_t v[32];
                tmem_ld16(tmem_addr(tY, 0, wg * 32) + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
                tmem_ld16(tmem_addr(tY, 0, wg * 32 + 16) + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
                tmem_wait_ld();
                if (j < len) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.y + (((size_t)b * sh.T + t0 + j) * sh.H + h) * kP + wg * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
                        w.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
                        w.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
                        w.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
                        dst[q] = w;
                    }
                }
            }
            fence_before_sync();
            if (__syncthreads_or(fail)) aborted = true;
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
bool tc_scan_supported(const Shape &sh, int dtype, const void *x, const void *B, const void *C, const void *y) {
    auto a16 = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
    return dtype == SSD_BF16 && sh.P == kP && (sh.N == 64 || sh.N == 128) && (sh.Q == 128 || sh.Q == 256) &&
           a16(x) && a16(B) && a16(C) && a16(y);
}

static int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

cudaError_t launch_chunk_scan_tc(const __nv_bfloat16 *x, const __nv_bfloat16 *B, const __nv_bfloat16 *C,
                                 const float *D, const float *s, const float *Sprev, __nv_bfloat16 *y, int *status,
                                 const Shape &sh, cudaStream_t st) {
    CUtensorMap mC, mB, mX;
    const uint64_t dbc[4] = {(uint64_t)sh.N, (uint64_t)sh.G, (uint64_t)sh.T, (uint64_t)sh.batch};
    const uint64_t sbc[3] = {(uint64_t)sh.N * 2, (uint64_t)sh.G * sh.N * 2, (uint64_t)sh.T * sh.G * sh.N * 2};
    const uint32_t box_bc[4] = {64, 1, kRows, 1};
    const uint64_t dx[4] = {(uint64_t)sh.P, (uint64_t)sh.H, (uint64_t)sh.T, (uint64_t)sh.batch};
    const uint64_t sx[3] = {(uint64_t)sh.P * 2, (uint64_t)sh.H * sh.P * 2, (uint64_t)sh.T * sh.H * sh.P * 2};
    const uint32_t box_x[4] = {64, 1, kRows, 1};
    if (!make_map_bf16(&mC, C, 4, dbc, sbc, box_bc) || !make_map_bf16(&mB, B, 4, dbc, sbc, box_bc) ||
        !make_map_bf16(&mX, x, 4, dx, sx, box_x))
        return cudaErrorInvalidValue;
    ScanParams p;
    p.sh = sh;
    p.s = s;
    p.Sprev = Sprev;
    p.D = D;
    p.y = y;
    p.status = status;
    p.NK = (sh.N + 63) / 64;
    p.halves = sh.Q / kRows;
    p.heads_per_unit = min(8, sh.heads_per_group);
    p.blocks_per_group = (sh.heads_per_group + p.heads_per_unit - 1) / p.heads_per_unit;
    p.n_units = sh.batch * sh.nc * p.halves * sh.G * p.blocks_per_group;
    cudaError_t e = cudaFuncSetAttribute(chunk_scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const int grid = min(p.n_units, sm_count());
    chunk_scan_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(mC, mB, mX, p);
    return cudaGetLastError();
}

}  // namespace ssd
