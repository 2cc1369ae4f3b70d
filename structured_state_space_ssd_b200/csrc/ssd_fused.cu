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
//  * Second-half units read S~_{c-1} from the ring and count themselves as
//    done with it; a first-half unit overwrites a slot only after every
//    second half up to the previous chunk has read (a count, since second
//    halves of different chunks finish in any order).  Every wait is
//    bounded: on expiry the status word is set to SSD_ERR_TIMEOUT and the
//    CTA finishes without waiting.
//
// Warp roles: each CTA runs two head pipelines side by side; pipeline pl
// takes every other head of a unit (units hold up to 4 heads).  Its eight
// CUDA-core warps (warps 8pl..8pl+7: two warpgroups, each covering the 128
// TMEM lanes and half of every tile's columns), its issuer warp (16 + pl;
// one lane issues TMA loads and tcgen05.mma) and its publisher warp (18 + pl;
// the GPU-scope fences and flags of the state hand-off) pass the pipeline's
// own X tile, state tile, decay mask (one 128-token K-half at a time) and
// accumulators back and forth through mbarriers, so that one pipeline's
// CUDA-core work overlaps the other's tensor-core products.  C, B and G are
// shared by the unit's heads.
#include "ssd_common.cuh"
#include "tc_prims.cuh"
#include "tma_host.h"

// Optional phase timestamps for performance work: compiled in only with
// -DSSD_TRACE, which also provides ssd_trace_buffer (one 32-slot record per
// head and pipeline).  Production builds contain no trace code.
#ifdef SSD_TRACE
__device__ unsigned long long *ssd_trace_buffer = nullptr;
#define SSD_TRACE_POINT(ev)                                                                                    \
    do {                                                                                                       \
        if (ssd_trace_buffer && wtid == 0 && trace_i < 30) {                                                   \
            unsigned long long t_;                                                                             \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                                           \
            ssd_trace_buffer[((size_t)blockIdx.x * 2 + pl) * 1024 + trace_i * 32 + (ev)] = t_;               \
        }                                                                                                      \
    } while (0)
#else
#define SSD_TRACE_POINT(ev) \
    do {                    \
    } while (0)
#endif
#ifdef SSD_TRACE
// waits until the values v[0..n) have arrived, then records event ev
#define SSD_TRACE_ARRIVED(v, n, ev)                              \
    do {                                                         \
        float acc_ = 0.f;                                        \
        for (int i_ = 0; i_ < (n); ++i_) acc_ += (v)[i_];        \
        if (acc_ == -1.2345e-30f) ssd_trace_buffer[0] = 1;       \
        SSD_TRACE_POINT(ev);                                     \
    } while (0)
#else
#define SSD_TRACE_ARRIVED(v, n, ev) \
    do {                            \
    } while (0)
#endif

namespace ssd {

using namespace tc;

namespace fz {

constexpr int kWgThreads = 128;                  // one warpgroup: the 128 TMEM lanes
constexpr int kPipeThreads = 2 * kWgThreads;     // two warpgroups per head pipeline, each half the columns
constexpr int kSimtWarps = 2 * kPipeThreads / 32;  // warps 0-15: CUDA-core work of pipelines 0 and 1
constexpr int kThreads = 2 * kPipeThreads + 128;  // + warps 16-17: issuers, 18-19: publishers
constexpr int kRows = 128;
constexpr int kP = 64;

// TMEM columns (512 allocated).  Pipeline pl owns D[pl], M[pl] and Y[pl].
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColG = 0;    // G: 128 (first half) or 256 (second half) fp32 columns
constexpr uint32_t kColD = 128;  // first half only: chunk-state accumulators, 64 columns per pipeline
constexpr uint32_t kColM = 256;  // decay mask (one 128-token K-half, bf16 pairs), 64 columns per pipeline
constexpr uint32_t kColY = 384;  // output accumulators, 64 columns per pipeline

// Shared memory (bytes from a 1 KiB-aligned base)
constexpr uint32_t kOffC = 0;                  // C rows of the half: 2 K-atoms x 128 rows x 128 B
constexpr uint32_t kOffB = 32768;              // B rows 0..Q-1: 2 K-atoms x 256 rows x 128 B
constexpr uint32_t kOffX = kOffB + 65536;      // per pipeline: X rows 0..Q-1, 256 rows x 128 B
constexpr uint32_t kOffS = kOffX + 2 * 32768;  // per pipeline: S~ tile (2 atoms x 64 rows x 128 B), or
                                               // the decayed X rows 0..127 before the chunk-state product
constexpr uint32_t kOffJ = kOffS + 2 * 16384;  // per pipeline, 2 buffers: s values (256 floats)
constexpr uint32_t kOffF = kOffJ + 4 * 1024;   // per pipeline, 2 buffers: column factors (256 floats)
constexpr uint32_t kSmemBytes = kOffF + 4 * 1024 + 1024;

constexpr uint32_t kFlagPolls = 1u << 22;

struct Params {
    Shape sh;
    const float *s;     // [b][H][nc][Q] per-chunk inclusive prefix sums of dt*A
    const float *D;     // [H]
    const float *init;  // [b][H][P][N] or null
    float *fin;         // [b][H][P][N] or null
    float *ring;        // [b][H][2][P][N]
    int *ready;         // [b*H]: chunks whose outgoing state is published
    int *cons;          // [b*H]: second halves that have read their entering state (a count: second
                        // halves of different chunks finish in any order)
    int *counter;       // unit dispenser
    int *status;
    __nv_bfloat16 *y;
    int NK;             // 64-wide K-atoms along N (C and the S~ tile)
    int halves;         // Q / 128
    int heads_per_unit;
    int blocks_per_group;
    int n_units;
};

// One head pipeline: its issuer warp and its warpgroup.  Barriers signalled
// once per head of the pipeline are waited with parity (use & 1), `use`
// counting the pipeline's earlier heads; both sides keep identical counters.
struct PipeBars {
    uint64_t x_full;      // X tile landed (TMA)
    uint64_t x_free;      // products reading the X tile done
    uint64_t j_full[2];   // s values landed (bulk copy), double-buffered
    uint64_t xd_full;     // first half: decayed X written (4 warp arrivals)
    uint64_t d_done;      // first half: chunk-state product done
    uint64_t s_full;      // S~ tile written (4 warp arrivals)
    uint64_t inter_done;  // inter-chunk product done
    uint64_t m_full;      // one mask K-half written (4 warp arrivals)
    uint64_t m_free;      // product reading it done
    uint64_t mx_done;     // every product of the head done
    uint64_t y_free;      // output accumulator drained (4 warp arrivals)
    uint64_t ring_done;   // ring stores issued (first half) / ring loads consumed (second half)
};

struct Bars {
    uint64_t cb;          // C and B tiles landed (TMA)
    uint64_t g_done;      // G = C B^T in TMEM
    uint64_t unit_full;   // unit id posted (issuer 0)
    uint64_t unit_empty;  // unit id read (16 CUDA-core warps, issuer 1, 2 publishers)
    uint64_t unit_done;   // both pipelines finished the unit (2 issuer arrivals)
    PipeBars pb[2];
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
// Each poll parks the warp for up to kSuspendNs, so the bound is about
// kWaitPolls * kSuspendNs (~2 s) of waiting, after which the status word
// records SSD_ERR_TIMEOUT.
constexpr uint32_t kSuspendNs = 100000;
constexpr uint32_t kWaitPolls = 20000;
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort, int *status) {
    if (mbar_try_wait(bar, parity)) return true;
    for (uint32_t i = 0; i < kWaitPolls; ++i) {
        if (mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
        if (*abort) return false;
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
        __nanosleep(64);
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
                     const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mY,
                     const fz::Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint8_t *sC = smem + kOffC;
    uint8_t *sB = smem + kOffB;
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
        uint64_t *all = reinterpret_cast<uint64_t *>(&bars);
        for (int i = 0; i < (int)(sizeof(Bars) / 8); ++i) mbar_init(&all[i], 1);
        mbar_init(&bars.unit_empty, kSimtWarps + 3);
        mbar_init(&bars.unit_done, 2);
        for (int q = 0; q < 2; ++q) {
            mbar_init(&bars.pb[q].xd_full, kPipeThreads / 32);
            mbar_init(&bars.pb[q].s_full, kPipeThreads / 32);
            mbar_init(&bars.pb[q].m_full, kPipeThreads / 32);
            mbar_init(&bars.pb[q].y_free, kPipeThreads / 32);
            mbar_init(&bars.pb[q].ring_done, kPipeThreads / 32);
        }
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;

    if (warp >= kSimtWarps + 2) {
        // ------------------------------------------------------------------
        // Publisher warps: warp 18 + pl makes pipeline pl's chain hand-offs
        // visible, so that neither the CUDA-core warps nor the issuer wait
        // for a GPU-scope release.  After a first half's ring stores it
        // releases `ready` (S~_c readable); after a second half consumed
        // S~_{c-1} it adds one to `cons` (the ring slot may be rewritten).
        // The warps' arrival on ring_done (a CTA-scope release, acquired by
        // this thread's wait) puts their accesses before this thread's
        // GPU-scope release, which carries them along (release is cumulative).
        // ------------------------------------------------------------------
        const int pl = warp - kSimtWarps - 2;
        PipeBars &pb = bars.pb[pl];
        uint32_t ucnt = 0, rcnt = 0;
        for (;;) {
            wait_bar(&bars.unit_full, par_of(ucnt), abort, p.status);
            ++ucnt;
            const int u = s_unit;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.unit_empty);
            if (u >= p.n_units) break;
            const Unit un = decode(u, p);
            if (un.row0 >= un.len) continue;
            const bool first = (un.r == 0);
            for (int h = un.h0 + pl; h < un.h1; h += 2, ++rcnt) {
                wait_bar(&pb.ring_done, par_of(rcnt), abort, p.status);
                if (lane == 0) {
                    const size_t bh = (size_t)un.b * sh.H + h;
                    if (first) {
                        if (un.c < sh.nc - 1) st_release_gpu(p.ready + bh, un.c + 1);
                    } else {
                        red_release_add_gpu(p.cons + bh, 1);
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp >= kSimtWarps) {
        // ------------------------------------------------------------------
        // Issuer warps: warp 16 drives pipeline 0 and also hands out units,
        // loads C/B and forms G; warp 17 drives pipeline 1.  The whole warp
        // follows the control flow and waits; lane 0 alone issues.
        // ------------------------------------------------------------------
        const int pl = warp - kSimtWarps;
        const bool leader = (lane == 0);
        PipeBars &pb = bars.pb[pl];
        uint8_t *sXp = smem + kOffX + pl * 32768;
        uint8_t *sSp = smem + kOffS + pl * 16384;
        float *sJp = reinterpret_cast<float *>(smem + kOffJ) + pl * 512;
        const uint32_t tY = tmem + kColY + pl * 64, tM = tmem + kColM + pl * 64, tD = tmem + kColD + pl * 64;
        if (leader && pl == 0) {
            tma_prefetch_desc(&mC);
            tma_prefetch_desc(&mB);
            tma_prefetch_desc(&mX);
        }
        uint32_t use = 0, r0use = 0, mcnt = 0, ucnt = 0, cbcnt = 0, units_done = 0;
        const uint32_t idG0 = idesc_bf16_f32(kRows, kRows, 0, 0);
        const uint32_t idG1 = idesc_bf16_f32(kRows, 2 * kRows, 0, 0);
        const uint32_t idInter = idesc_bf16_f32(kRows, kP, 0, 0);
        const uint32_t idState = idesc_bf16_f32(kRows, kP, 1, 1);
        const uint32_t idMX = idesc_bf16_f32(kRows, kP, 0, 1);
        for (;;) {
            int u = 0;
            if (pl == 0) {
                if (ucnt > 0) wait_bar(&bars.unit_empty, par_of(ucnt - 1), abort, p.status);
                if (leader) {
                    u = atomicAdd(p.counter, 1);
                    s_unit = u;
                    mbar_arrive(&bars.unit_full);
                }
                u = __shfl_sync(0xffffffffu, u, 0);
            } else {
                wait_bar(&bars.unit_full, par_of(ucnt), abort, p.status);
                u = s_unit;
                __syncwarp();
                if (leader) mbar_arrive(&bars.unit_empty);
            }
            ++ucnt;
            if (u >= p.n_units) break;
            const Unit un = decode(u, p);
            if (un.row0 >= un.len) continue;
            const bool first = (un.r == 0);
            const int qbox = Q / kRows;
            if (pl == 0) {
                // both pipelines are done with the previous unit's C, B and G
                if (units_done > 0) wait_bar(&bars.unit_done, par_of(units_done - 1), abort, p.status);
                if (leader) {
                    mbar_arrive_expect_tx(&bars.cb, (uint32_t)(NK + 2 * qbox) * 16384u);
                    for (int k = 0; k < NK; ++k)
                        tma_load_4d(sC + k * 16384, &mC, &bars.cb, k * 64, un.g, un.t0 + un.row0, un.b);
                    for (int k = 0; k < 2; ++k)
                        for (int q = 0; q < qbox; ++q)
                            tma_load_4d(sB + k * 32768 + q * 16384, &mB, &bars.cb, k * 64, un.g,
                                        un.t0 + q * kRows, un.b);
                }
            }
            ++units_done;
            wait_bar(&bars.cb, par_of(cbcnt++), abort, p.status);
            fence_after_sync();
            if (pl == 0) {
                // G = C_r B^T  (rows of this half x columns 0 .. end of this half)
                if (leader) {
                    for (int kk = 0; kk < NK * 4; ++kk) {
                        const int atom = kk >> 2, kin = kk & 3;
                        mma_ss(tmem + kColG, smem_desc_sw128(smem_u32(sC) + atom * 16384 + kin * 32, 16, 1024),
                               smem_desc_sw128(smem_u32(sB) + atom * 32768 + kin * 32, 16, 1024),
                               first ? idG0 : idG1, kk > 0);
                    }
                    mma_commit(&bars.g_done);
                }
                __syncwarp();
            }
            bool any = false;
            for (int h = un.h0 + pl; h < un.h1; h += 2, ++use) {
                any = true;
                const int jb = use & 1;
                // this head's X rows 0..Q-1 and s values; warm L2 for the pipeline's next head
                if (use > 0) wait_bar(&pb.x_free, par_of(use - 1), abort, p.status);
                if (leader) {
                    mbar_arrive_expect_tx(&pb.x_full, (uint32_t)qbox * 16384u);
                    for (int q = 0; q < qbox; ++q)
                        tma_load_4d(sXp + q * 16384, &mX, &pb.x_full, 0, h, un.t0 + q * kRows, un.b);
                    mbar_arrive_expect_tx(&pb.j_full[jb], (uint32_t)Q * 4u);
                    bulk_load(sJp + jb * 256, p.s + (((size_t)un.b * sh.H + h) * sh.nc + un.c) * Q,
                              (uint32_t)Q * 4u, &pb.j_full[jb]);
                    if (h + 2 < un.h1)
                        for (int q = 0; q < qbox; ++q) tma_prefetch_4d(&mX, 0, h + 2, un.t0 + q * kRows, un.b);
                }
                __syncwarp();
                if (first) {
                    // stage 2: D = B_c^T (decayed X), M = n (128), N = p, K = Q tokens; the decayed
                    // rows 0..127 sit in the S~ buffer, rows 128.. were decayed in place
                    wait_bar(&pb.xd_full, par_of(r0use), abort, p.status);
                    fence_after_sync();
                    if (leader) {
                        for (int kk = 0; kk < Q / 16; ++kk) {
                            const uint32_t xb = (kk < 8) ? smem_u32(sSp) + kk * 2048 : smem_u32(sXp) + kk * 2048;
                            mma_ss(tD, smem_desc_sw128(smem_u32(sB) + kk * 2048, 32768, 1024),
                                   smem_desc_sw128(xb, 16, 1024), idState, kk > 0);
                        }
                        mma_commit(&pb.d_done);
                    }
                    __syncwarp();
                    ++r0use;
                }
                // stage 4 product: Y = C_r S~^T
                wait_bar(&pb.s_full, par_of(use), abort, p.status);
                if (use > 0) wait_bar(&pb.y_free, par_of(use - 1), abort, p.status);
                fence_after_sync();
                if (leader) {
                    for (int kk = 0; kk < NK * 4; ++kk) {
                        const int atom = kk >> 2, kin = kk & 3;
                        mma_ss(tY, smem_desc_sw128(smem_u32(sC) + atom * 16384 + kin * 32, 16, 1024),
                               smem_desc_sw128(smem_u32(sSp) + atom * 8192 + kin * 32, 16, 1024), idInter, kk > 0);
                    }
                    mma_commit(&pb.inter_done);
                }
                __syncwarp();
                // stage 1 product: Y += M X, one 128-token K-half at a time
                const int nhalf = first ? 1 : 2;
                for (int hf = 0; hf < nhalf; ++hf) {
                    wait_bar(&pb.m_full, par_of(mcnt), abort, p.status);
                    if (hf == 0 && !first) wait_bar(&pb.x_full, par_of(use), abort, p.status);
                    fence_after_sync();
                    if (leader) {
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ts(tY, tM + kk * 8, smem_desc_sw128(smem_u32(sXp) + (hf * 8 + kk) * 2048, 16, 1024),
                                   idMX, 1);
                        mma_commit(&pb.m_free);
                    }
                    __syncwarp();
                    ++mcnt;
                }
                if (leader) {
                    mma_commit(&pb.mx_done);
                    mma_commit(&pb.x_free);
                }
                __syncwarp();
            }
            // this pipeline is done with the unit once its last products completed
            if (any) wait_bar(&pb.mx_done, par_of(use - 1), abort, p.status);
            if (leader) mbar_arrive(&bars.unit_done);
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------------
        // CUDA-core warps: warps 8pl..8pl+7 serve pipeline pl as two
        // warpgroups; warpgroup `half` takes columns [32 half, 32 half + 32)
        // of every 64-wide tile and every other 32-column slab of the mask.
        // ------------------------------------------------------------------
        const int pl = warp >> 3;
        const int half = (warp >> 2) & 1;
        const int wtid = tid & (kPipeThreads - 1);
        const int lrow = ((warp & 3) << 5) + lane;  // TMEM lane = row within the chunk half
        const uint32_t lane_base = (uint32_t)((warp & 3) << 5) << 16;
        const int wg_bar = 1 + pl;
        PipeBars &pb = bars.pb[pl];
        uint8_t *sXp = smem + kOffX + pl * 32768;
        uint8_t *sSp = smem + kOffS + pl * 16384;
        float *sJp = reinterpret_cast<float *>(smem + kOffJ) + pl * 512;
        float *sFp = reinterpret_cast<float *>(smem + kOffF) + pl * 512;
        const uint32_t tY = tmem + kColY + pl * 64, tM = tmem + kColM + pl * 64, tD = tmem + kColD + pl * 64;
        uint32_t use = 0, r0use = 0, mcnt = 0, ucnt = 0, gcnt = 0;
#ifdef SSD_TRACE
        int trace_i = 0;
#endif
        for (;;) {
            wait_bar(&bars.unit_full, par_of(ucnt), abort, p.status);
            ++ucnt;
            const int u = s_unit;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.unit_empty);
            if (u >= p.n_units) break;
            const Unit un = decode(u, p);
            if (un.row0 >= un.len) {
                // no rows: count the (unread) entering state of every head as read
                if (tid == 0)
                    for (int h = un.h0; h < un.h1; ++h) red_release_add_gpu(p.cons + un.b * sh.H + h, 1);
                continue;
            }
            const bool first = (un.r == 0);
            const int j = un.row0 + lrow;  // this thread's row within the chunk
            const int kcols = un.row0 + kRows;
            wait_bar(&bars.g_done, par_of(gcnt++), abort, p.status);
            for (int h = un.h0 + pl; h < un.h1; h += 2, ++use) {
                const int jb = use & 1;
                float *sJb = sJp + jb * 256;
                float *sFb = sFp + jb * 256;
                const size_t bh = (size_t)un.b * sh.H + h;
                const size_t PN = (size_t)kP * N;
                SSD_TRACE_POINT(0);
                // the previous head's y tile left the S~ buffer before it is overwritten (the
                // stores are issued by the pipeline's last thread, never by the thread that
                // fences and publishes states, whose GPU-scope fence would wait for them)
                if (wtid == kPipeThreads - 1) bulk_wait_read();
                SSD_TRACE_POINT(1);
                wait_bar(&pb.j_full[jb], par_of(use >> 1), abort, p.status);
                for (int i = wtid; i < kcols; i += kPipeThreads) sFb[i] = expf(sJb[i | 31] - sJb[i]);
                named_bar_sync(wg_bar, kPipeThreads);
                SSD_TRACE_POINT(2);
                const float *src = (un.c == 0) ? (p.init ? p.init + bh * PN : nullptr)
                                               : p.ring + (bh * 2 + ((un.c - 1) & 1)) * PN;
                const float sj = sJb[j];
                const float Dh = p.D[h];
                const float s_end = sJb[Q - 1];

                // decay mask for 32-column slabs sl = half, half + 2 of K-half hf, into TMEM, in
                // 16-column pieces (few live registers: the entering state may be in flight)
                auto mask_half = [&](int hf) {
#pragma unroll 1
                    for (int sl = half; sl < 4; sl += 2) {
                        const int i0 = hf * 128 + sl * 32;
                        uint32_t o[16];
                        if (i0 > j) {
#pragma unroll
                            for (int q = 0; q < 16; ++q) o[q] = 0u;
                            tmem_st16(tM + sl * 16 + lane_base, o);
                            continue;
                        }
                        uint32_t g[32];
                        tmem_ld16(tmem + kColG + i0 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&g[0]));
                        tmem_ld16(tmem + kColG + i0 + 16 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&g[16]));
                        tmem_wait_ld();
                        if (i0 + 31 < j) {
                            // below the diagonal block: row factor x column factor, both <= 1
                            const float rf = expf(sj - sJb[i0 + 31]);
                            const float4 *f4 = reinterpret_cast<const float4 *>(sFb + i0);
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const float4 f = f4[q];
                                const float2 w0 = mul_f32x2(make_float2(rf, rf), make_float2(f.x, f.y));
                                const float2 w1 = mul_f32x2(make_float2(rf, rf), make_float2(f.z, f.w));
                                const float2 m0 = mul_f32x2(
                                    make_float2(__uint_as_float(g[4 * q]), __uint_as_float(g[4 * q + 1])), w0);
                                const float2 m1 = mul_f32x2(
                                    make_float2(__uint_as_float(g[4 * q + 2]), __uint_as_float(g[4 * q + 3])), w1);
                                o[2 * q] = pack_bf16x2(m0.x, m0.y);
                                o[2 * q + 1] = pack_bf16x2(m1.x, m1.y);
                            }
                        } else {
                            // the diagonal 32x32 block: one exponential per element
#pragma unroll
                            for (int q = 0; q < 16; ++q) {
                                const int ia = i0 + 2 * q, ib = ia + 1;
                                float a = (ia <= j) ? __uint_as_float(g[2 * q]) * expf(sj - sJb[ia]) : 0.f;
                                float bb = (ib <= j) ? __uint_as_float(g[2 * q + 1]) * expf(sj - sJb[ib]) : 0.f;
                                if (ia == j) a += Dh;
                                if (ib == j) bb += Dh;
                                o[q] = pack_bf16x2(a, bb);
                            }
                        }
                        tmem_st16(tM + sl * 16 + lane_base, o);
                    }
                    tmem_wait_st();
                };
                // Y *= exp(s_j) (stage 4's decay from the chunk start), then hand mask K-half 0 to
                // the issuer: its product accumulates onto the scaled Y
                auto scale_and_release_mask = [&]() {
                    wait_bar(&pb.inter_done, par_of(use), abort, p.status);
                    fence_after_sync();
                    const float e = expf(sj);
                    uint32_t v[32];
                    tmem_ld16(tY + half * 32 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
                    tmem_ld16(tY + half * 32 + 16 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 32; ++q) v[q] = __float_as_uint(__uint_as_float(v[q]) * e);
                    tmem_st16(tY + half * 32 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
                    tmem_st16(tY + half * 32 + 16 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
                    tmem_wait_st();
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pb.m_full);
                    ++mcnt;
                };

                if (first) {
                    // x_i * exp(s_end - s_i) for the chunk state: rows 0..127 into the S~ buffer
                    // (rows 0..127 of the X tile stay undecayed for the masked product), rows 128.. in place
                    wait_bar(&pb.x_full, par_of(use), abort, p.status);
                    SSD_TRACE_POINT(21);
#pragma unroll 1
                    for (int base = wtid; base < Q * 8; base += 4 * kPipeThreads) {
                        uint4 v[4];
                        float w[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const int idx = min(base + r * kPipeThreads, Q * 8 - 1);
                            v[r] = *reinterpret_cast<const uint4 *>(sXp + idx * 16);
                            w[r] = expf(s_end - sJb[idx >> 3]);
                        }
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const int idx = base + r * kPipeThreads;
                            if (idx >= Q * 8) continue;
                            uint4 o;
                            o.x = pack_bf16x2(bf16lo(v[r].x) * w[r], bf16hi(v[r].x) * w[r]);
                            o.y = pack_bf16x2(bf16lo(v[r].y) * w[r], bf16hi(v[r].y) * w[r]);
                            o.z = pack_bf16x2(bf16lo(v[r].z) * w[r], bf16hi(v[r].z) * w[r]);
                            o.w = pack_bf16x2(bf16lo(v[r].w) * w[r], bf16hi(v[r].w) * w[r]);
                            *reinterpret_cast<uint4 *>(((idx >> 3) < kRows ? sSp : sXp) + idx * 16) = o;
                        }
                    }
                    fence_view_async_shared();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pb.xd_full);
                    SSD_TRACE_POINT(3);
                    // mask K-half 0 (the whole K range of a first half) while the state product runs
                    // and before waiting on the chain, so that the chain's path holds no mask work
                    if (mcnt > 0) wait_bar(&pb.m_free, par_of(mcnt - 1), abort, p.status);
                    SSD_TRACE_POINT(22);
                    fence_after_sync();
                    mask_half(0);
                    // S~_{c-1} must be published and the outgoing ring slot free of readers: the slot
                    // held S~_{c-2}, read by the second half of chunk c-1, so wait until the second
                    // halves of chunks 0..c-1 have all read theirs
                    if (wtid == 0) {
                        if (un.c > 0) wait_flag(p.ready + bh, un.c, abort, p.status);
                        if (p.halves == 2 && un.c >= 2) wait_flag(p.cons + bh, un.c, abort, p.status);
                    }
                    named_bar_sync(wg_bar, kPipeThreads);
                    SSD_TRACE_POINT(15);
                    // this thread's 32 columns of S~_{c-1} (lane n; [p][n] like the initial state)
                    const int n = lrow;
                    float old[32];
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        old[q] = (src && n < N) ? __ldcg(src + (size_t)(half * 32 + q) * N + n) : 0.f;
                    SSD_TRACE_POINT(4);
                    SSD_TRACE_ARRIVED(old, 32, 8);
                    // stage 3: S~_c = exp(s_end) S~_{c-1} + S_c; S~_{c-1} in bf16 is this head's
                    // inter-chunk operand (the decayed rows left the S~ buffer with the state product)
                    wait_bar(&pb.d_done, par_of(r0use), abort, p.status);
                    ++r0use;
                    named_bar_sync(wg_bar, kPipeThreads);
                    fence_after_sync();
                    SSD_TRACE_POINT(5);
                    {
                        // the outgoing state goes to the ring or, after the last chunk, to the final state
                        const float dchunk = expf(s_end);
                        float *dst = (un.c == sh.nc - 1) ? (p.fin ? p.fin + bh * PN : nullptr)
                                                         : p.ring + (bh * 2 + (un.c & 1)) * PN;
#pragma unroll
                        for (int q0 = 0; q0 < 32; q0 += 16) {
                            uint32_t dv[16];
                            tmem_ld16(tmem + kColD + pl * 64 + half * 32 + q0 + lane_base, dv);
                            tmem_wait_ld();
                            if (n < N && dst) {
#pragma unroll
                                for (int q = 0; q < 16; ++q)
                                    __stcg(dst + (size_t)(half * 32 + q0 + q) * N + n,
                                           fmaf(dchunk, old[q0 + q], __uint_as_float(dv[q])));
                            }
                        }
                        // the publisher warp releases the stores
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&pb.ring_done);
                        // S~_{c-1} in bf16 into column n of the S~ tile ([p][n], 128-byte swizzled)
                        if (n < N) {
                            uint8_t *srow = sSp + (n >> 6) * 8192;
                            const int chunk = (n & 63) >> 3, sub = (n & 7) * 2;
#pragma unroll
                            for (int q = 0; q < 32; ++q) {
                                const int pp = half * 32 + q;
                                *reinterpret_cast<__nv_bfloat16 *>(srow + pp * 128 + ((chunk ^ (pp & 7)) << 4) + sub) =
                                    __float2bfloat16_rn(old[q]);
                            }
                        }
                    }
                    SSD_TRACE_POINT(12);
                    fence_view_async_shared();
                    named_bar_sync(wg_bar, kPipeThreads);
                    SSD_TRACE_POINT(13);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pb.s_full);
                    SSD_TRACE_POINT(6);
                    scale_and_release_mask();
                    SSD_TRACE_POINT(7);
                } else {
                    // mask K-half 0 first, then wait for the entering state (chunk 0 reads the
                    // initial state)
                    if (mcnt > 0) wait_bar(&pb.m_free, par_of(mcnt - 1), abort, p.status);
                    fence_after_sync();
                    mask_half(0);
                    if (wtid == 0 && un.c > 0) wait_flag(p.ready + bh, un.c, abort, p.status);
                    named_bar_sync(wg_bar, kPipeThreads);
                    // this thread's pieces of S~_{c-1} ([p][n]: 8 consecutive n of one row p each)
                    const int nchunks = kP * NK * 8;
                    float4 lo[4], hi[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int idx = wtid + r * kPipeThreads;
                        const int pr = idx / (NK * 8), n = (idx % (NK * 8)) * 8;
                        lo[r] = hi[r] = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (idx < nchunks && src && n < N) {
                            lo[r] = __ldcg(reinterpret_cast<const float4 *>(src + (size_t)pr * N + n));
                            hi[r] = __ldcg(reinterpret_cast<const float4 *>(src + (size_t)pr * N + n + 4));
                        }
                    }
                    SSD_TRACE_POINT(3);
                    SSD_TRACE_ARRIVED(reinterpret_cast<const float *>(lo), 16, 8);
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int idx = wtid + r * kPipeThreads;
                        const int pr = idx / (NK * 8), n = (idx % (NK * 8)) * 8;
                        if (idx >= nchunks) continue;
                        uint4 v;
                        v.x = pack_bf16x2(lo[r].x, lo[r].y);
                        v.y = pack_bf16x2(lo[r].z, lo[r].w);
                        v.z = pack_bf16x2(hi[r].x, hi[r].y);
                        v.w = pack_bf16x2(hi[r].z, hi[r].w);
                        *reinterpret_cast<uint4 *>(sSp + (n >> 6) * 8192 + pr * 128 +
                                                   ((((n & 63) >> 3) ^ (pr & 7)) << 4)) = v;
                    }
                    // the publisher warp releases the ring slot: this warp's loads are consumed
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pb.ring_done);
                    fence_view_async_shared();
                    named_bar_sync(wg_bar, kPipeThreads);
                    if (lane == 0) mbar_arrive(&pb.s_full);
                    SSD_TRACE_POINT(6);
                    scale_and_release_mask();
                    SSD_TRACE_POINT(7);
                    // mask K-half 1 once the product of K-half 0 has read the mask buffer
                    wait_bar(&pb.m_free, par_of(mcnt - 1), abort, p.status);
                    fence_after_sync();
                    mask_half(1);
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pb.m_full);
                    ++mcnt;
                }
                SSD_TRACE_POINT(9);
                // stage 5: y = bf16(Y), staged in the S~ buffer (its inter-chunk product is done)
                // in the 128-byte-swizzled layout and written by one TMA store
                wait_bar(&pb.mx_done, par_of(use), abort, p.status);
                SSD_TRACE_POINT(10);
                fence_after_sync();
                {
                    uint32_t v[32];
                    tmem_ld16(tY + half * 32 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
                    tmem_ld16(tY + half * 32 + 16 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
                    tmem_wait_ld();
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pb.y_free);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
                        w.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
                        w.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
                        w.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
                        const int qq = half * 4 + q;  // 16-byte chunk of the 128-byte row
                        *reinterpret_cast<uint4 *>(sSp + lrow * 128 + ((qq ^ (lrow & 7)) << 4)) = w;
                    }
                    fence_view_async_shared();
                    named_bar_sync(wg_bar, kPipeThreads);
                    if (wtid == kPipeThreads - 1) {
                        tma_store_4d(&mY, sSp, 0, h, un.t0 + un.row0, un.b);
                        bulk_commit();
                    }
                }
                SSD_TRACE_POINT(11);
#ifdef SSD_TRACE
                if (ssd_trace_buffer && wtid == 0 && trace_i < 30)
                    ssd_trace_buffer[((size_t)blockIdx.x * 2 + pl) * 1024 + trace_i * 32 + 14] =
                        ((unsigned long long)h << 32) | ((unsigned long long)un.c << 8) | (first ? 1 : 0);
                ++trace_i;
#endif
            }
        }
    }
    if (warp < kSimtWarps && (tid & (kPipeThreads - 1)) == kPipeThreads - 1) bulk_wait_all();
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
    CUtensorMap mY;
    if (!make_map_bf16(&mC, C, 4, dbc, sbc, box_bc) || !make_map_bf16(&mB, B, 4, dbc, sbc, box_bc) ||
        !make_map_bf16(&mX, x, 4, dx, sx, box_x) || !make_map_bf16(&mY, y, 4, dx, sx, box_x))
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
    p.heads_per_unit = min(4, sh.heads_per_group);
    p.blocks_per_group = (sh.heads_per_group + p.heads_per_unit - 1) / p.heads_per_unit;
    p.n_units = sh.nc * sh.batch * sh.G * p.blocks_per_group * p.halves;
    cudaError_t e =
        cudaFuncSetAttribute(ssd_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const int grid = min(p.n_units, device_sm_count());
    ssd_fused_kernel<<<grid, kThreads, kSmemBytes, st>>>(mC, mB, mX, mY, p);
    return cudaGetLastError();
}

}  // namespace ssd
