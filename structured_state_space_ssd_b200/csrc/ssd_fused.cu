// ssd_fused.cu -- the bf16 SSD forward as one persistent tensor-core kernel.
//
// "Transformers are SSMs" (analysis page, section "The Block-Decomposition SSD
// Algorithm") computes the layer in stages: the quadratic masked form inside
// each chunk of Q tokens (stage 1), chunk-final states (stage 2), the scalar
// recurrence of those states across chunks (stage 3), the inter-chunk output
// (stage 4) and the sum (stage 5).  This kernel runs stages 1-5 for every
// chunk, every head and both 128-row halves of a chunk without sending the
// fp32 chunk states through HBM:
//
//  * A work unit is (chunk c, batch b, group g, block of heads, half r).
//    Units are handed out by an atomic counter in chunk-major order, so a
//    unit only ever waits for units handed out before it (which are running
//    or done): there is no deadlock however many CTAs are resident.
//  * First-half units (rows 0..127) own the chunk state: per head they form
//    S_c = B_c^T (exp(s_end - s_i) x_i) on the tensor cores (stage 2), wait
//    for the state S~_{c-1} entering the chunk (published by the first-half
//    unit of chunk c-1), publish S~_c = exp(s_end) S~_{c-1} + S_c (stage 3)
//    into a two-slot fp32 ring that stays in L2, and write final_state for
//    the last chunk.
//  * Every unit then produces its 128 output rows per head: G = C_r B^T once
//    per unit into TMEM, Y = exp(s_j) C_r S~_{c-1}^T (stage 4), the causal
//    decay mask M = G o exp(s_j - s_i) (+ D_h on the diagonal) written by the
//    CUDA cores into TMEM as the bf16 A operand, Y += M X (stage 1), y = bf16(Y)
//    (stage 5).
//  * Second-half units read S~_{c-1} from the ring and then release the
//    slot; a first-half unit overwrites a slot only after both readers of its
//    previous content are done.  Every wait is bounded: on expiry the status
//    word is set to SSD_ERR_TIMEOUT and the CTA finishes without waiting.
//
// Warp roles: warps 0-7 (two warpgroups, each covering the 128 TMEM lanes) do
// the CUDA-core work; one lane of warp 8 issues TMA loads and tcgen05.mma.
// They hand buffers to each other through mbarriers: X tiles and chunk-state
// accumulators are double-buffered per head, as are the output accumulators,
// and the decay mask is split in two K-halves so that masking one half
// overlaps the tensor-core product of the other.
#include "ssd_common.cuh"
#include "tc_prims.cuh"
#include "tma_host.h"

namespace ssd {

using namespace tc;

namespace fz {

constexpr int kSimtThreads = 256;
constexpr int kThreads = kSimtThreads + 32;
constexpr int kIssuerWarp = 8;
constexpr int kSimtBar = 1;  // named barrier of the CUDA-core warps
constexpr int kRows = 128;
constexpr int kP = 64;

// TMEM columns (512 allocated)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColG = 0;    // G: 128 (first half) or 256 (second half) fp32 columns
constexpr uint32_t kColD = 128;  // first half: chunk-state accumulators D[2], 64 columns each
constexpr uint32_t kColM = 256;  // decay mask, bf16 pairs: K-half 0 at +0, K-half 1 at +64
constexpr uint32_t kColY = 384;  // output accumulators Y[2], 64 columns each

// Shared memory (bytes from a 1 KiB-aligned base)
constexpr uint32_t kOffC = 0;                 // C rows of the half: 2 K-atoms x 128 rows x 128 B
constexpr uint32_t kOffB = 32768;             // B rows 0..Q-1: 2 K-atoms x 256 rows x 128 B
constexpr uint32_t kOffX = kOffB + 65536;     // X tiles: 2 buffers x 256 rows x 128 B
constexpr uint32_t kOffX0 = kOffX + 65536;    // first half: X rows 0..127, undecayed
constexpr uint32_t kOffS = kOffX0 + 16384;    // S~ as bf16 K-major: 2 buffers x 2 atoms x 64 rows x 128 B
constexpr uint32_t kOffJ = kOffS + 32768;     // s values: 2 buffers x 256 floats
constexpr uint32_t kOffF = kOffJ + 2048;      // column factors: 2 buffers x 256 floats
constexpr uint32_t kSmemBytes = kOffF + 2048 + 1024;

constexpr uint32_t kBarPolls = 1u << 22;
constexpr uint32_t kFlagPolls = 1u << 22;

struct Params {
    Shape sh;
    const float *s;     // [b][H][nc][Q] per-chunk inclusive prefix sums of dt*A
    const float *D;     // [H]
    const float *init;  // [b][H][P][N] or null
    float *fin;         // [b][H][P][N] or null
    float *ring;        // [b][H][2][P][N]
    int *ready;         // [b*H]: chunks whose outgoing state is published
    int *cons;          // [b*H]: chunks whose second half has read its entering state
    int *counter;       // unit dispenser
    int *status;
    __nv_bfloat16 *y;
    int NK;             // 64-wide K-atoms along N (C and the S~ tile)
    int halves;         // Q / 128
    int heads_per_unit;
    int blocks_per_group;
    int n_units;
};

struct Bars {
    uint64_t cb;             // C and B tiles landed (TMA)
    uint64_t x_full[2];      // X tile landed (TMA)
    uint64_t x_free[2];      // last MMA reading an X tile done
    uint64_t x0_full;        // undecayed X rows 0..127 landed (TMA)
    uint64_t x0_free;        // MMA reading them done
    uint64_t xd_full;        // decayed X written (8 warp arrivals); first-half heads only
    uint64_t d_done;         // chunk-state product done; first-half heads only
    uint64_t s_full[2];      // S~ tile written (8 warp arrivals)
    uint64_t inter_done[2];  // inter-chunk product done
    uint64_t m_full[2];      // mask K-half written (8 warp arrivals)
    uint64_t m_free[2];      // MMA reading a mask K-half done
    uint64_t mx_done[2];     // all products of a head done
    uint64_t y_free[2];      // output accumulator drained (8 warp arrivals)
    uint64_t unit_full;      // unit id posted (issuer)
    uint64_t unit_empty;     // unit id read (8 warp arrivals)
};

struct Unit {
    int b, c, g, h0, h1, r, t0, len, row0;
};

__device__ __forceinline__ Unit decode(int u, const Params &p) {
    Unit un;
    int rem = u;
    un.r = rem % p.halves;
    rem /= p.halves;
    const int hb = rem % p.blocks_per_group;
    rem /= p.blocks_per_group;
    un.g = rem % p.sh.G;
    rem /= p.sh.G;
    un.b = rem % p.sh.batch;
    un.c = rem / p.sh.batch;
    un.h0 = un.g * p.sh.heads_per_group + hb * p.heads_per_unit;
    un.h1 = min(un.h0 + p.heads_per_unit, (un.g + 1) * p.sh.heads_per_group);
    un.t0 = un.c * p.sh.Q;
    un.len = min(p.sh.Q, p.sh.T - un.t0);
    un.row0 = un.r * kRows;
    return un;
}

__device__ __forceinline__ uint8_t *align_1k(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Bounded mbarrier wait that gives up at once after any wait in the CTA failed.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort, int *status) {
    for (uint32_t i = 0; i < kBarPolls; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && *abort) return false;
    }
    atomicExch(status, SSD_ERR_TIMEOUT);
    *abort = 1;
    return false;
}

// Bounded wait for a GPU-scope counter to reach `target` (acquire).
__device__ __forceinline__ bool wait_flag(const int *flag, int target, volatile int *abort, int *status) {
    for (uint32_t i = 0; i < kFlagPolls; ++i) {
        if (ld_acquire_gpu(flag) >= target) return true;
        if (*abort || ld_relaxed_gpu(status) != 0) {
            *abort = 1;
            return false;
        }
        __nanosleep(128);
    }
    atomicExch(status, SSD_ERR_TIMEOUT);
    *abort = 1;
    return false;
}

__device__ __forceinline__ uint32_t par_of(uint32_t use) { return use & 1u; }

}  // namespace fz

using namespace fz;

__global__ void __launch_bounds__(fz::kThreads, 1)
    ssd_fused_kernel(const __grid_constant__ CUtensorMap mC, const __grid_constant__ CUtensorMap mB,
                     const __grid_constant__ CUtensorMap mX, const fz::Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint8_t *sC = smem + kOffC;
    uint8_t *sB = smem + kOffB;
    uint8_t *sX = smem + kOffX;
    uint8_t *sX0 = smem + kOffX0;
    uint8_t *sS = smem + kOffS;
    float *sJ = reinterpret_cast<float *>(smem + kOffJ);
    float *sF = reinterpret_cast<float *>(smem + kOffF);
    __shared__ Bars bars;
    __shared__ uint32_t tslot;
    __shared__ int s_unit;
    __shared__ int s_abort;
    volatile int *abort = &s_abort;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const Shape sh = p.sh;
    const int Q = sh.Q, N = sh.N, NK = p.NK;

    if (warp == 0) tmem_alloc(&tslot, kTmemCols);
    if (tid == 0) {
        s_abort = 0;
        // Phases: a barrier signalled once per head is waited with parity (use & 1),
        // where `use` counts the heads that signalled it before; the two roles
        // keep identical counters.
        uint64_t *all = reinterpret_cast<uint64_t *>(&bars);
        for (int i = 0; i < (int)(sizeof(Bars) / 8); ++i) mbar_init(&all[i], 1);
        // CUDA-core arrivals: one per warp
        uint64_t *eight[] = {&bars.xd_full,   &bars.s_full[0], &bars.s_full[1], &bars.m_full[0],
                             &bars.m_full[1], &bars.y_free[0], &bars.y_free[1], &bars.unit_empty};
        for (int i = 0; i < 8; ++i) mbar_init(eight[i], 8);
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;

    if (warp == kIssuerWarp) {
        // ------------------------------------------------------------------
        // TMA / MMA issue: the whole warp follows the control flow and waits;
        // lane 0 alone issues loads, products and commits.
        // ------------------------------------------------------------------
        const bool leader = (lane == 0);
        if (leader) {
            tma_prefetch_desc(&mC);
            tma_prefetch_desc(&mB);
            tma_prefetch_desc(&mX);
        }
        uint32_t kh = 0, ucnt = 0, x0cnt = 0, cbcnt = 0;
        uint32_t mcnt[2] = {0, 0};
        const uint32_t idG0 = idesc_bf16_f32(kRows, kRows, 0, 0);
        const uint32_t idG1 = idesc_bf16_f32(kRows, 2 * kRows, 0, 0);
        const uint32_t idInter = idesc_bf16_f32(kRows, kP, 0, 0);
        const uint32_t idState = idesc_bf16_f32(kRows, kP, 1, 1);
        const uint32_t idMX = idesc_bf16_f32(kRows, kP, 0, 1);
        for (;;) {
            if (ucnt > 0) wait_bar(&bars.unit_empty, par_of(ucnt - 1), abort, p.status);
            int u = 0;
            if (leader) {
                u = atomicAdd(p.counter, 1);
                s_unit = u;
                mbar_arrive(&bars.unit_full);
            }
            u = __shfl_sync(0xffffffffu, u, 0);
            ++ucnt;
            if (u >= p.n_units) break;
            const Unit un = decode(u, p);
            if (un.row0 >= un.len) continue;
            const bool first = (un.r == 0);
            // the previous unit's products must be done before its operands are replaced
            if (kh > 0) wait_bar(&bars.mx_done[(kh - 1) & 1], par_of((kh - 1) >> 1), abort, p.status);
            const int qbox = Q / kRows;
            if (leader) {
                mbar_arrive_expect_tx(&bars.cb, (uint32_t)(NK + 2 * qbox) * 16384u);
                for (int k = 0; k < NK; ++k)
                    tma_load_4d(sC + k * 16384, &mC, &bars.cb, k * 64, un.g, un.t0 + un.row0, un.b);
                for (int k = 0; k < 2; ++k)
                    for (int q = 0; q < qbox; ++q)
                        tma_load_4d(sB + k * 32768 + q * 16384, &mB, &bars.cb, k * 64, un.g, un.t0 + q * kRows,
                                    un.b);
            }
            wait_bar(&bars.cb, par_of(cbcnt++), abort, p.status);
            fence_after_sync();
            // G = C_r B^T  (rows of this half x columns 0 .. end of this half)
            if (leader)
                for (int kk = 0; kk < NK * 4; ++kk) {
                    const int atom = kk >> 2, kin = kk & 3;
                    mma_ss(tmem + kColG, smem_desc_sw128(smem_u32(sC) + atom * 16384 + kin * 32, 16, 1024),
                           smem_desc_sw128(smem_u32(sB) + atom * 32768 + kin * 32, 16, 1024), first ? idG0 : idG1,
                           kk > 0);
                }
            __syncwarp();
            for (int h = un.h0; h < un.h1; ++h, ++kh) {
                const int buf = kh & 1;
                const uint32_t use = kh >> 1;
                uint8_t *sXb = sX + buf * 32768;
                uint8_t *sSb = sS + buf * 16384;
                const uint32_t tY = tmem + kColY + buf * 64;
                // X rows 0..Q-1 of head h
                if (kh >= 2) wait_bar(&bars.x_free[buf], par_of(use - 1), abort, p.status);
                if (leader) {
                    mbar_arrive_expect_tx(&bars.x_full[buf], (uint32_t)qbox * 16384u);
                    for (int q = 0; q < qbox; ++q)
                        tma_load_4d(sXb + q * 16384, &mX, &bars.x_full[buf], 0, h, un.t0 + q * kRows, un.b);
                }
                if (first) {
                    if (x0cnt > 0) wait_bar(&bars.x0_free, par_of(x0cnt - 1), abort, p.status);
                    if (leader) {
                        mbar_arrive_expect_tx(&bars.x0_full, 16384u);
                        tma_load_4d(sX0, &mX, &bars.x0_full, 0, h, un.t0, un.b);
                    }
                    // stage 2: D = B_c^T (decayed X), M = n (128), N = p, K = Q tokens
                    wait_bar(&bars.xd_full, par_of(x0cnt), abort, p.status);
                    fence_after_sync();
                    if (leader) {
                        const uint32_t tD = tmem + kColD + buf * 64;
                        for (int kk = 0; kk < Q / 16; ++kk)
                            mma_ss(tD, smem_desc_sw128(smem_u32(sB) + kk * 2048, 32768, 1024),
                                   smem_desc_sw128(smem_u32(sXb) + kk * 2048, 16, 1024), idState, kk > 0);
                        mma_commit(&bars.d_done);
                        mma_commit(&bars.x_free[buf]);
                    }
                    __syncwarp();
                }
                // stage 4 product: Y = C_r S~^T
                wait_bar(&bars.s_full[buf], par_of(use), abort, p.status);
                if (kh >= 2) wait_bar(&bars.y_free[buf], par_of(use - 1), abort, p.status);
                fence_after_sync();
                if (leader) {
                    for (int kk = 0; kk < NK * 4; ++kk) {
                        const int atom = kk >> 2, kin = kk & 3;
                        mma_ss(tY, smem_desc_sw128(smem_u32(sC) + atom * 16384 + kin * 32, 16, 1024),
                               smem_desc_sw128(smem_u32(sSb) + atom * 8192 + kin * 32, 16, 1024), idInter, kk > 0);
                    }
                    mma_commit(&bars.inter_done[buf]);
                }
                __syncwarp();
                // stage 1 product: Y += M X, one K-half (128 tokens) at a time
                const int nhalf = first ? 1 : 2;
                for (int hf = 0; hf < nhalf; ++hf) {
                    wait_bar(&bars.m_full[hf], par_of(mcnt[hf]), abort, p.status);
                    if (hf == 0) {
                        if (first)
                            wait_bar(&bars.x0_full, par_of(x0cnt), abort, p.status);
                        else
                            wait_bar(&bars.x_full[buf], par_of(use), abort, p.status);
                    }
                    fence_after_sync();
                    if (leader) {
                        const uint32_t xbase = first ? smem_u32(sX0) : smem_u32(sXb) + hf * 16384;
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ts(tY, tmem + kColM + hf * 64 + kk * 8, smem_desc_sw128(xbase + kk * 2048, 16, 1024),
                                   idMX, 1);
                        mma_commit(&bars.m_free[hf]);
                    }
                    __syncwarp();
                    ++mcnt[hf];
                }
                if (leader) {
                    mma_commit(&bars.mx_done[buf]);
                    mma_commit(first ? &bars.x0_free : &bars.x_free[buf]);
                }
                __syncwarp();
                if (first) ++x0cnt;
            }
        }
    } else {
        // ------------------------------------------------------------------
        // CUDA-core warps
        // ------------------------------------------------------------------
        const int wg = warp >> 2;                         // warpgroup: which 32 of the 64 columns
        const int lrow = ((warp & 3) << 5) + lane;        // TMEM lane = row within the half
        const uint32_t lane_base = (uint32_t)((warp & 3) << 5) << 16;
        uint32_t kh = 0, ucnt = 0, r0cnt = 0;
        uint32_t mcnt[2] = {0, 0};
        for (;;) {
            wait_bar(&bars.unit_full, par_of(ucnt), abort, p.status);
            ++ucnt;
            const int u = s_unit;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.unit_empty);
            if (u >= p.n_units) break;
            const Unit un = decode(u, p);
            if (un.row0 >= un.len) {
                // no rows: release the (unread) entering state of every head for the slot's next writer
                if (tid == 0)
                    for (int h = un.h0; h < un.h1; ++h) st_release_gpu(p.cons + un.b * sh.H + h, un.c + 1);
                continue;
            }
            const bool first = (un.r == 0);
            const int j = un.row0 + lrow;  // this thread's row within the chunk
            for (int h = un.h0; h < un.h1; ++h, ++kh) {
                const int buf = kh & 1;
                const uint32_t use = kh >> 1;
                float *sJb = sJ + buf * 256;
                float *sFb = sF + buf * 256;
                uint8_t *sXb = sX + buf * 32768;
                uint8_t *sSb = sS + buf * 16384;
                const uint32_t tY = tmem + kColY + buf * 64;
                const size_t bh = (size_t)un.b * sh.H + h;
                const float *sc = p.s + (bh * sh.nc + un.c) * Q;
                for (int i = tid; i < Q; i += kSimtThreads) sJb[i] = sc[i];
                named_bar_sync(kSimtBar, kSimtThreads);
                const int kcols = un.row0 + kRows;
                for (int i = tid; i < kcols; i += kSimtThreads) sFb[i] = expf(sJb[i | 31] - sJb[i]);

                if (first) {
                    // decay X rows in place for the chunk state: x_i * exp(s_end - s_i)
                    wait_bar(&bars.x_full[buf], par_of(use), abort, p.status);
                    const float s_end = sJb[Q - 1];
                    for (int idx = tid; idx < Q * 8; idx += kSimtThreads) {
                        const int i = idx >> 3;
                        const float w = expf(s_end - sJb[i]);
                        uint4 *ptr = reinterpret_cast<uint4 *>(sXb + idx * 16);
                        uint4 v = *ptr;
                        v.x = pack_bf16x2(bf16lo(v.x) * w, bf16hi(v.x) * w);
                        v.y = pack_bf16x2(bf16lo(v.y) * w, bf16hi(v.y) * w);
                        v.z = pack_bf16x2(bf16lo(v.z) * w, bf16hi(v.z) * w);
                        v.w = pack_bf16x2(bf16lo(v.w) * w, bf16hi(v.w) * w);
                        *ptr = v;
                    }
                    fence_view_async_shared();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars.xd_full);
                    // stage 3: S~_c = exp(s_end) S~_{c-1} + S_c
                    if (tid == 0) {
                        if (un.c > 0) wait_flag(p.ready + bh, un.c, abort, p.status);
                        if (p.halves == 2 && un.c >= 2) wait_flag(p.cons + bh, un.c, abort, p.status);
                    }
                    wait_bar(&bars.d_done, par_of(r0cnt), abort, p.status);
                    ++r0cnt;
                    named_bar_sync(kSimtBar, kSimtThreads);
                    fence_after_sync();
                    {
                        const float dchunk = expf(s_end);
                        const int n = lrow;
                        const uint32_t tD = tmem + kColD + buf * 64 + wg * 32;
                        uint32_t dv[32];
                        tmem_ld16(tD + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&dv[0]));
                        tmem_ld16(tD + 16 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&dv[16]));
                        tmem_wait_ld();
                        if (n < N) {
                            const size_t PN = (size_t)kP * N;
                            const float *src = (un.c == 0) ? p.init : p.ring + (bh * 2 + ((un.c - 1) & 1)) * PN;
                            float *dst = (un.c == sh.nc - 1) ? p.fin : p.ring + (bh * 2 + (un.c & 1)) * PN;
                            if (un.c == 0 && src) src += bh * PN;
                            if (un.c == sh.nc - 1 && dst) dst += bh * PN;
                            uint8_t *srow = sSb + (n >> 6) * 8192;
                            const int chunk = (n & 63) >> 3, sub = (n & 7) * 2;
#pragma unroll 4
                            for (int q = 0; q < 32; ++q) {
                                const int pp = wg * 32 + q;
                                const float old = src ? __ldcg(src + (size_t)pp * N + n) : 0.f;
                                const float nw = fmaf(dchunk, old, __uint_as_float(dv[q]));
                                if (dst) __stcg(dst + (size_t)pp * N + n, nw);
                                *reinterpret_cast<__nv_bfloat16 *>(srow + pp * 128 + ((chunk ^ (pp & 7)) << 4) + sub) =
                                    __float2bfloat16_rn(old);
                            }
                        }
                    }
                    __threadfence();
                    fence_view_async_shared();
                    named_bar_sync(kSimtBar, kSimtThreads);
                    if (tid == 0 && un.c < sh.nc - 1) st_release_gpu(p.ready + bh, un.c + 1);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars.s_full[buf]);
                } else {
                    // entering state S~_{c-1} -> bf16 K-major tile
                    if (tid == 0 && un.c > 0) wait_flag(p.ready + bh, un.c, abort, p.status);
                    named_bar_sync(kSimtBar, kSimtThreads);
                    const size_t PN = (size_t)kP * N;
                    const float *src = (un.c == 0) ? (p.init ? p.init + bh * PN : nullptr)
                                                   : p.ring + (bh * 2 + ((un.c - 1) & 1)) * PN;
                    for (int idx = tid; idx < kP * NK * 8; idx += kSimtThreads) {
                        const int pr = idx / (NK * 8), n = (idx % (NK * 8)) * 8;
                        uint4 v = make_uint4(0, 0, 0, 0);
                        if (src && n < N) {
                            const float4 a = __ldcg(reinterpret_cast<const float4 *>(src + (size_t)pr * N + n));
                            const float4 bq = __ldcg(reinterpret_cast<const float4 *>(src + (size_t)pr * N + n + 4));
                            v.x = pack_bf16x2(a.x, a.y);
                            v.y = pack_bf16x2(a.z, a.w);
                            v.z = pack_bf16x2(bq.x, bq.y);
                            v.w = pack_bf16x2(bq.z, bq.w);
                        }
                        *reinterpret_cast<uint4 *>(sSb + (n >> 6) * 8192 + pr * 128 + ((((n & 63) >> 3) ^ (pr & 7)) << 4)) =
                            v;
                    }
                    fence_view_async_shared();
                    named_bar_sync(kSimtBar, kSimtThreads);
                    if (tid == 0) st_release_gpu(p.cons + bh, un.c + 1);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars.s_full[buf]);
                }

                // Y *= exp(s_j): stage 4's decay from the chunk start
                wait_bar(&bars.inter_done[buf], par_of(use), abort, p.status);
                fence_after_sync();
                const float sj = sJb[j];
                {
                    const float e = expf(sj);
                    uint32_t v[16];
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const uint32_t ta = tY + wg * 32 + hf * 16 + lane_base;
                        tmem_ld16(ta, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int q = 0; q < 16; ++q) v[q] = __float_as_uint(__uint_as_float(v[q]) * e);
                        tmem_st16(ta, v);
                    }
                }
                // decay mask into TMEM, one K-half of 128 columns at a time
                const float Dh = p.D[h];
                const int nhalf = first ? 1 : 2;
                for (int hf = 0; hf < nhalf; ++hf) {
                    if (mcnt[hf] > 0) wait_bar(&bars.m_free[hf], par_of(mcnt[hf] - 1), abort, p.status);
                    fence_after_sync();
                    for (int sl = wg; sl < 4; sl += 2) {
                        const int i0 = hf * 128 + sl * 32;
                        uint32_t gv[32];
                        tmem_ld16(tmem + kColG + i0 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&gv[0]));
                        tmem_ld16(tmem + kColG + i0 + 16 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&gv[16]));
                        tmem_wait_ld();
                        uint32_t o[16];
                        if (i0 + 31 < j) {
                            const float rf = expf(sj - sJb[i0 + 31]);
#pragma unroll
                            for (int q = 0; q < 16; ++q) {
                                const float a = __uint_as_float(gv[2 * q]) * (rf * sFb[i0 + 2 * q]);
                                const float bb = __uint_as_float(gv[2 * q + 1]) * (rf * sFb[i0 + 2 * q + 1]);
                                o[q] = pack_bf16x2(a, bb);
                            }
                        } else if (i0 > j) {
#pragma unroll
                            for (int q = 0; q < 16; ++q) o[q] = 0u;
                        } else {
#pragma unroll
                            for (int q = 0; q < 16; ++q) {
                                const int ia = i0 + 2 * q, ib = ia + 1;
                                float a = (ia <= j) ? __uint_as_float(gv[2 * q]) * expf(sj - sJb[ia]) : 0.f;
                                float bb = (ib <= j) ? __uint_as_float(gv[2 * q + 1]) * expf(sj - sJb[ib]) : 0.f;
                                if (ia == j) a += Dh;
                                if (ib == j) bb += Dh;
                                o[q] = pack_bf16x2(a, bb);
                            }
                        }
                        tmem_st16(tmem + kColM + hf * 64 + (sl * 32) / 2 + lane_base, o);
                    }
                    tmem_wait_st();
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars.m_full[hf]);
                    ++mcnt[hf];
                }
                // stage 5: y = bf16(Y)
                wait_bar(&bars.mx_done[buf], par_of(use), abort, p.status);
                fence_after_sync();
                {
                    uint32_t v[32];
                    tmem_ld16(tY + wg * 32 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
                    tmem_ld16(tY + wg * 32 + 16 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
                    tmem_wait_ld();
                    if (j < un.len) {
                        uint4 *dst = reinterpret_cast<uint4 *>(
                            p.y + (((size_t)un.b * sh.T + un.t0 + j) * sh.H + h) * kP + wg * 32);
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
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.y_free[buf]);
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
bool fused_supported(const Shape &sh, int dtype) {
    return dtype == SSD_BF16 && sh.P == kP && (sh.N == 64 || sh.N == 128) && (sh.Q == 128 || sh.Q == 256);
}

static int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

cudaError_t launch_ssd_fused(const __nv_bfloat16 *x, const __nv_bfloat16 *B, const __nv_bfloat16 *C,
                             const float *D, const float *s, const float *init, float *fin, float *ring, int *ready,
                             int *cons, int *counter, int *status, __nv_bfloat16 *y, const Shape &sh,
                             cudaStream_t st) {
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
    Params p;
    p.sh = sh;
    p.s = s;
    p.D = D;
    p.init = init;
    p.fin = fin;
    p.ring = ring;
    p.ready = ready;
    p.cons = cons;
    p.counter = counter;
    p.status = status;
    p.y = y;
    p.NK = (sh.N + 63) / 64;
    p.halves = sh.Q / kRows;
    p.heads_per_unit = min(8, sh.heads_per_group);
    p.blocks_per_group = (sh.heads_per_group + p.heads_per_unit - 1) / p.heads_per_unit;
    p.n_units = sh.nc * sh.batch * sh.G * p.blocks_per_group * p.halves;
    cudaError_t e =
        cudaFuncSetAttribute(ssd_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const int grid = min(p.n_units, device_sm_count());
    ssd_fused_kernel<<<grid, kThreads, kSmemBytes, st>>>(mC, mB, mX, p);
    return cudaGetLastError();
}

}  // namespace ssd
