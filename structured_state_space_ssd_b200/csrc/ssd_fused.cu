// ssd_fused.cu -- the bf16 SSD forward as one persistent tensor-core kernel.
//
// "Transformers are SSMs" (analysis page, section "The Block-Decomposition SSD
// Algorithm") computes the layer in stages: chunk prefix sums of the
// log-decay (stage 0), the quadratic masked form inside each chunk of Q
// tokens (stage 1), chunk-final states (stage 2), the scalar recurrence of
// those states across chunks (stage 3), the inter-chunk output (stage 4) and
// the sum (stage 5).  This kernel runs every stage in one launch; nothing but
// the chained states (L2-resident: fp32, and bf16 operand tiles of them)
// leaves the SM.
//
// Blocks of 128 rows.  A chunk of Q = 256 tokens is two blocks, and the
// second block reaches the first through the state at the chunk's midpoint
// instead of through the off-diagonal block of the quadratic form: the same
// block decomposition applied once more inside the chunk, so the function is
// unchanged and only the diagonal 128 x 128 blocks of the semiseparable
// matrix are ever formed.  With s the inclusive prefix sum of dt*A from the
// chunk start, r the block's first row (s_{-1} = 0) and x~_i the rows
// scaled by a decay:
//
//   entering state  E   = exp(s_{r-1}) S~_{c-1} + B_{<r}^T (exp(s_{r-1} - s_i) x_i)
//   output          y_j = exp(s_j - s_{r-1}) C_j E^T
//                         + sum_{r <= i <= j} exp(s_j - s_i) (C_j . B_i) x_i + D_h x_j
//   chunk state     S~_c = exp(s_end - s_{r-1}) E + B_{>=r}^T (exp(s_end - s_i) x_i)   (last block)
//
//  * A work unit is (chunk c, batch b, group g, block of heads, block r).
//    Units are handed out by an atomic counter in an order (see decode) in
//    which a unit only ever waits for units handed out before it: there is
//    no deadlock however many CTAs are resident.
//  * The last block of a chunk owns the chunk state: it waits for S~_{c-1}
//    (published by the owner of chunk c-1), forms E and S~_c, and writes
//    S~_c over S~_{c-1} in its sequence's fp32 slot (or final_state after
//    the last chunk).  The other block of the next chunk needs S~_c only as
//    the bf16 operand of its inter-chunk product, so the owner also writes
//    that tile in the operand's layout and its publisher stores it with TMA
//    into a three-slot ring, from which the other block's issuer loads it
//    with TMA (no CUDA-core work); a tile slot is overwritten only after its
//    reader has counted itself done.  On long sequences (kD = 4) the owners
//    also publish their local states L_c early and start from the most recent
//    published S~_j of the 4 chunks before, folding in the L after it (a
//    decoupled look-back; see fused_lookback), and the other blocks read the
//    fp32 S~ from those slots too.  Every wait on another CTA is
//    bounded: on expiry the status word is set to SSD_ERR_TIMEOUT and the
//    waits that follow give up at once (the CTA's own barriers are still
//    waited for, so nothing it issued is in flight when it exits).
//  * A launch covers 64 head columns and up to 128 state columns: P = 128 and
//    N = 256 run as two launches each (the second state half adds to y;
//    kAccum), a head below 64 columns is zero-padded.  With kGated the drain
//    applies the block's gate and a per-head GroupNorm instead of storing y.
//
// Warp roles: two head pipelines per CTA, pipeline pl taking every other head
// of a unit.  Its eight CUDA-core warps (two warpgroups over the 128 TMEM
// lanes) form the prefix sums, scale x, build the decay mask, move the states
// and drain the accumulators; its issuer warp (16 + pl) loads x with TMA and
// issues tcgen05.mma; its publisher warp (18 + pl) makes the state hand-offs
// visible to other CTAs (and stores an owner's bf16 state tile).  C, B and
// G = C B^T (the block's 128 x 128) are shared by the unit's heads; an owner's
// units hold half as many heads as the other block's, whose heads take about
// half as long.
#include <algorithm>

#include "ssd_common.cuh"
#include "tc_prims.cuh"
#include "tma_host.h"

namespace ssd {

using namespace tc;

namespace fz {

constexpr int kRows = 128;                         // rows of a block: one TMEM lane each
constexpr int kP = 64;                             // head dimension of this path
constexpr int kPipeThreads = 256;                  // two warpgroups per head pipeline
constexpr int kPipeWarps = kPipeThreads / 32;
constexpr int kSimtWarps = 2 * kPipeWarps;         // warps 0-15: CUDA-core work of pipelines 0 and 1
constexpr int kThreads = 32 * kSimtWarps + 128;    // + warps 16-17: issuers, 18-19: publishers
constexpr float kLog2e = 1.4426950408889634f;

// TMEM columns (512 allocated).  G is the unit's C B^T block (fp32).  Per
// pipeline: accumulator A holds the pre-block state, then the inter-chunk
// product; accumulator B holds the block's own state contribution, then the
// masked product; M holds the bf16 decay mask (the A operand of M X).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColG = 0;
__device__ __forceinline__ uint32_t col_acc_a(int pl) { return 128u + 192u * pl; }
__device__ __forceinline__ uint32_t col_acc_b(int pl) { return 192u + 192u * pl; }
__device__ __forceinline__ uint32_t col_mask(int pl) { return 256u + 192u * pl; }

// Shared memory, from a 1 KiB-aligned base.  Tiles are bf16 rows of 128 bytes
// in the 128-byte-swizzled layout TMA writes (8-row atoms of 1 KiB).
constexpr uint32_t kOffC = 0;           // C rows of the block: NK atoms x 128 rows
constexpr uint32_t kOffB = 32768;       // B rows 0..Q-1: 2 atoms of 256 rows (atom stride 32 KiB)
constexpr uint32_t kOffPipe = 98304;    // per pipeline: x rows 0..127 | W | x rows 128..255, 16 KiB each
constexpr uint32_t kPipeBytes = 49152;  // W: scaled x rows, then an owner's bf16 state tile or the y tile
constexpr uint32_t kOffAux = kOffPipe + 2 * kPipeBytes;
constexpr uint32_t kAuxFloats = 256 + 256 + 16;  // per pipeline: s (log2 units), column factors, warp totals
constexpr uint32_t kOffStat = kOffAux + 2 * kAuxFloats * 4;  // gated drain: per pipeline, half, row (mean, M2)
constexpr uint32_t kOffWB = kOffStat + 2 * 2 * kRows * 8;      // gated drain: per pipeline, the head's weight, bias
constexpr uint32_t kSmemBytes = kOffWB + 2 * 2 * kP * 4 + 1024;

constexpr uint32_t kDefaultFlagPolls = 1u << 22;

struct Params {
    Shape sh;
    const float *dt;    // [b][T][H]
    const float *A;     // [H]
    const float *D;     // [H]
    const float *init;  // [b][H][P][N] or null
    float *fin;         // [b][H][P][N] or null
    // The chain (see fused_lookback; the depth D is the kernel's template argument).  fp32 states, each
    // [P/4][N][4] (see ring_quad): with D = 1 one slot per sequence holding the latest S~ (only owners
    // read it, each in place before writing its own); with look-back chunk c's S~_c and L_c in slot c % R.
    // The other blocks read S~_{c-1} as a bf16 tile (tensor map mR: [b*H*R][tile_rows][64], slot c % R,
    // the 128-byte swizzle of the stage-4 operand), stored by the owner's publisher with TMA.
    float *ring;        // [b*H][1 or R][1 or 2][P/4][N][4]
    int tile_rows;      // rows of a bf16 state tile: N rounded up to 64 (the K extent of stage 4)
    int *inc;           // c + 1 once S~_c is published: [b*H] without look-back, [b*H][R] with (inc_flag)
    int *tin;           // [b*H][R]: c + 1 once the bf16 tile of S~_c is in slot c % R (tiles may land out of order)
    int *agg;           // [b*H][R]: c + 1 once L_c and sigma_c are published (look-back only)
    int *cons;          // [b*H][R]: reads of the slot so far, every use (a count)
    float *sig;         // [b*H][R]: sigma_c, chunk c's total decay in log2 units (look-back only)
    int *counter;       // unit dispenser
    int *status;
    __nv_bfloat16 *y;   // y + p_off (row stride p_full); read back only by the second state half
    int NK;             // 64-wide K-atoms along N
    int halves;         // Q / 128
    // Units of row block r hold up to hpu[r] heads of a group (blocks[r] units per group, units[r] =
    // batch * G * blocks[r] per chunk): the owners' block (r = 1) does more per head, so its units
    // are smaller, which keeps unit lengths alike.  With one block per chunk r = 0 only.
    int hpu[2];
    int blocks[2];
    int units[2];
    int n_units;
    uint32_t flag_polls;  // bound of each wait on another CTA's flag
    int withhold_bh;      // test hook: the owner of (b*H + h, chunk) below never publishes (-1: none)
    int withhold_c;
    // A state dimension of 256 runs as two launches over n = 0..127 and 128..255 (the state splits
    // into independent halves, y into the sum of their contributions): sh.N is the half's size,
    // state_ld the caller's n stride, n_off the half's first n; the second launch has no D skip
    // (D == null) and adds its result to the y the first one wrote (kernel template argument).
    int state_ld;
    int n_off;
    // Gated output (kernel template argument kGated): out = GroupNorm(y * silu(z)) with a group per head
    // (its 64 channels), written through the y tensor map in y's place; y itself is not written.
    const __nv_bfloat16 *z;  // [b][T][H][64]
    const float *gw, *gb;    // [H * 64] or null (1, 0)
    float eps;
    // The tile is 64 columns of p wide: a head dimension below 64 is zero-padded (x loads past P read
    // zero, y stores past P are clipped, state rows past P are neither read nor written), and P = 128
    // runs as two launches over columns p_off = 0 and 64 (the rows of the state are independent).
    int p_full;
    int p_off;
};

// One head pipeline.  Barriers signalled once per head of the pipeline are
// waited with parity (count & 1); both sides keep identical counters.
struct PipeBars {
    uint64_t x_full;     // x rows landed (TMA)
    uint64_t xd_full;    // owner: scaled x rows written (8 warp arrivals)
    uint64_t d_done;     // owner: state products done
    uint64_t m_full;     // decay mask written (8 warp arrivals)
    uint64_t s_full;     // entering-state tile written, state accumulators read (8 warp arrivals)
    uint64_t mx_done;    // every product of the head done
    uint64_t acc_free;   // accumulators drained (8 warp arrivals)
    uint64_t e_full;     // another block's entering-state tile landed (TMA from the bf16 ring)
    uint64_t t_free;     // owner: its bf16 state tile (in x rows 0..127) read by the publisher's TMA store
};

struct Bars {
    uint64_t cb;          // C and B tiles landed (TMA)
    uint64_t g_done;      // G = C B^T in TMEM
    uint64_t unit_full;   // unit id posted (issuer 0)
    uint64_t unit_empty;  // unit id read (16 CUDA-core warps, issuer 1, 2 publishers)
    uint64_t unit_done;   // both pipelines finished the unit's products (2 issuer arrivals)
    PipeBars pb[2];
};

struct Unit {
    int b, c, g, h0, h1, r, t0, len, row0;
    bool rows;   // the block has rows (the last chunk may be short)
    bool owner;  // the chunk's last block with rows: it carries the chunk state
};

// Hand-out order.  With one row block per chunk (Q = 128) units go chunk by chunk.  With two, the
// block owning chunk c's state (the last one) is handed out one step ahead of chunk c-1's other block:
//   [owners of chunk 0] [owners of 1, others of 0] [owners of 2, others of 1] ... [others of nc-1]
// so that the owners, which carry the inter-chunk chain, run ahead of the blocks that wait for it.
// Every unit still waits only for units handed out before it: an owner waits for the owners of the
// D chunks before (earlier steps) and for the readers of the slot it overwrites, chunk c-R's (the
// owners up to chunk c-R+D and the other block of chunk c-R+1, handed out with the owners of c-R+2, at
// least one step earlier as R >= 3; without look-back only the tile slot is counted, by its publisher);
// another block waits for the owner of the chunk before (two steps earlier).  So there is no deadlock
// however many CTAs are resident.
__device__ __forceinline__ Unit decode(int u, const Params &p) {
    Unit un;
    const int Mo = p.units[0], Mw = p.units[1];
    int idx;
    if (p.halves == 1) {
        un.r = 0;
        un.c = u / Mo;
        idx = u % Mo;
    } else if (u < Mw) {
        un.r = 1;
        un.c = 0;
        idx = u;
    } else {
        const int v = u - Mw, t = v / (Mw + Mo), j = v % (Mw + Mo);
        if (t < p.sh.nc - 1 && j < Mw) {
            un.r = 1;
            un.c = t + 1;
            idx = j;
        } else {
            un.r = 0;
            un.c = t;
            idx = (t < p.sh.nc - 1) ? j - Mw : j;
        }
    }
    const int hb = idx % p.blocks[un.r];
    idx /= p.blocks[un.r];
    un.g = idx % p.sh.G;
    un.b = idx / p.sh.G;
    un.h0 = un.g * p.sh.heads_per_group + hb * p.hpu[un.r];
    un.h1 = min(un.h0 + p.hpu[un.r], (un.g + 1) * p.sh.heads_per_group);
    un.t0 = un.c * p.sh.Q;
    un.len = min(p.sh.Q, p.sh.T - un.t0);
    un.row0 = un.r * kRows;
    un.rows = un.row0 < un.len;
    un.owner = un.rows && un.r == ((un.len - 1) >> 7);
    return un;
}

__device__ __forceinline__ uint8_t *align_1k(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Wait on one of the CTA's own mbarriers.  Its producers are this CTA's own
// warps, TMA and tensor cores, which always finish, so the wait is never cut
// short by a timeout on another CTA's flag.  The bound (about 2 s) only turns
// a defect of the kernel itself into a status instead of a hang; once one such
// wait has expired (`broken`), the CTA's later waits give up after about 1 ms
// so that the kernel still ends in bounded time.
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint64_t kBrokenWaitNs = 1000000ull;
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void wait_bar(uint64_t *bar, uint32_t parity, int *status, volatile int *broken) {
    if (mbar_try_wait(bar, parity)) return;
    const uint64_t t0 = global_ns(), limit = *broken ? kBrokenWaitNs : kWaitNs;
    for (;;) {
        if (mbar_try_wait(bar, parity)) return;
        if (global_ns() - t0 > limit) break;
    }
    atomicExch(status, SSD_ERR_TIMEOUT);
    *broken = 1;
}

// Bounded wait for another CTA's counter to reach `target` (acquire).  Gives
// up at once when a wait anywhere has already given up.
__device__ __forceinline__ void wait_flag(const int *flag, int target, uint32_t polls, volatile int *abort,
                                          int *status) {
    if (*abort) return;
    for (uint32_t i = 0; i < polls; ++i) {
        if (ld_acquire_gpu(flag) >= target) return;
        if (ld_relaxed_gpu(status) != 0) {
            *abort = 1;
            return;
        }
        __nanosleep(64);
    }
    atomicExch(status, SSD_ERR_TIMEOUT);
    *abort = 1;
}

__device__ __forceinline__ uint32_t par(uint32_t n) { return n & 1u; }

__device__ __forceinline__ uint4 lds128(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ void sts128(uint8_t *p, uint4 v) { *reinterpret_cast<uint4 *>(p) = v; }

// Byte offset of 16-byte chunk `chunk` of row `row` in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    return (uint32_t)row * 128u + ((uint32_t)(chunk ^ (row & 7)) << 4);
}

// The fp32 chunk states in the ring are stored in quads of p: entry (n, p) of
// a slot sits at float4 index (p / 4) * N + n, component p % 4.  A warp's 32
// lanes (32 consecutive n, one TMEM lane each) then move 512 contiguous bytes
// per 16-byte access.
__device__ __forceinline__ size_t ring_quad(int N, int n, int quad) { return (size_t)quad * N + n; }

// The flag that publishes S~_c of sequence bh.  Without look-back owners publish in chunk order, so
// one count per sequence serves (it reads c + 1 once S~_0 .. S~_c are out; a count measured faster
// here than a flag per slot); with look-back they may publish out of order: one flag per ring slot.
template <int kD>
__device__ __forceinline__ int *inc_flag(int *inc, int bh, int c) {
    constexpr int R = kD == 1 ? 3 : 2 * kD;
    return kD == 1 ? inc + bh : inc + bh * R + c % R;
}

// Eight bf16 scaled by w (fp32 products, one rounding to bf16).
__device__ __forceinline__ uint4 scale_bf16x8(uint4 v, float w) {
    const float2 ww = make_float2(w, w);
    uint4 o;
    float2 a;
    a = mul_f32x2(make_float2(bf16lo(v.x), bf16hi(v.x)), ww);
    o.x = pack_bf16x2(a.x, a.y);
    a = mul_f32x2(make_float2(bf16lo(v.y), bf16hi(v.y)), ww);
    o.y = pack_bf16x2(a.x, a.y);
    a = mul_f32x2(make_float2(bf16lo(v.z), bf16hi(v.z)), ww);
    o.z = pack_bf16x2(a.x, a.y);
    a = mul_f32x2(make_float2(bf16lo(v.w), bf16hi(v.w)), ww);
    o.w = pack_bf16x2(a.x, a.y);
    return o;
}

}  // namespace fz

using namespace fz;

// kAccum: the second half of a 256-wide state, which adds its y to the first half's.
// kD: the chain's look-back depth D (1: every owner waits for the chunk before).
// kGated: the drain applies the gate and the per-head GroupNorm (Params::z) and stores that instead of y.
template <bool kAccum, int kD, bool kGated>
__global__ void __launch_bounds__(fz::kThreads, 1)
    ssd_fused_kernel(const __grid_constant__ CUtensorMap mC, const __grid_constant__ CUtensorMap mB,
                     const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mY,
                     const __grid_constant__ CUtensorMap mR, const fz::Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint8_t *sC = smem + kOffC;
    uint8_t *sB = smem + kOffB;
    __shared__ Bars bars;
    __shared__ uint32_t tslot;
    __shared__ int s_unit;
    __shared__ int s_abort, s_broken;
    // per pipeline, for its publisher: warps that finished an owner's state stores (8 per head), and the
    // reads of another block's entering state (its issuer's tile load, 1 per head; with look-back its
    // warps' reads of the fp32 slot, 8 per head)
    __shared__ uint32_t s_owned[2], s_copied[2], s_agg[2];
    __shared__ int s_base[2];  // per pipeline: the chunk whose S~ the owner starts from (-1: initial state)
    volatile int *abort = &s_abort;
    volatile int *broken = &s_broken;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const Shape sh = p.sh;
    const int N = sh.N, NK = p.NK;
    constexpr int R = kD == 1 ? 3 : 2 * kD;  // ring slots per sequence (see fused_ring_slots)

    if (warp == 0) tmem_alloc(&tslot, kTmemCols);
    if (tid == 0) {
        s_abort = 0;
        s_broken = 0;
        s_owned[0] = s_owned[1] = s_copied[0] = s_copied[1] = s_agg[0] = s_agg[1] = 0;
        uint64_t *all = reinterpret_cast<uint64_t *>(&bars);
        for (int i = 0; i < (int)(sizeof(Bars) / 8); ++i) mbar_init(&all[i], 1);
        mbar_init(&bars.unit_empty, kSimtWarps + 3);
        mbar_init(&bars.unit_done, 2);
        for (int q = 0; q < 2; ++q) {
            mbar_init(&bars.pb[q].xd_full, kPipeWarps);
            mbar_init(&bars.pb[q].m_full, kPipeWarps);
            mbar_init(&bars.pb[q].s_full, kPipeWarps);
            mbar_init(&bars.pb[q].acc_free, kPipeWarps);
        }
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    // launched as a programmatic dependent of the workspace clear: everything above overlapped it; no
    // thread touches global memory before the clear has completed and its stores are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp >= kSimtWarps + 2) {
        // ------------------------------------------------------------------
        // Publisher warps: warp 18 + pl makes pipeline pl's hand-offs visible
        // to other CTAs, so that neither the CUDA-core warps nor the issuer
        // wait for a GPU-scope release.  After an owner's stores of L_c it
        // releases `agg` (look-back only); after its store of S~_c it releases
        // `inc` and adds one to `cons` of each slot it may have read, then
        // stores the bf16 tile of S~_c with TMA (once the slot's earlier
        // readers are done) and releases `tin`, so that the chain of owners
        // never waits for the tile; once another block has read S~_{c-1} it
        // adds one to that slot's `cons`.  The warps signal through CTA-scope release
        // counts in shared memory, acquired here by every lane, which puts
        // their stores before the lanes' GPU-scope releases (release is
        // cumulative).
        // ------------------------------------------------------------------
        const int pl = warp - kSimtWarps - 2;
        const uint8_t *sTile = smem + kOffPipe + pl * kPipeBytes + 16384;  // the owner's tile, in W
        uint32_t ucnt = 0, ocnt = 0, tcnt = 0, acnt = 0;
        // bounded wait for one of this pipeline's shared-memory counts to reach `target`
        auto wait_count = [&](const uint32_t *cnt, uint32_t target) {
            if (ld_acquire_cta_shared(cnt) >= target) return;
            const uint64_t t0 = global_ns(), limit = *broken ? kBrokenWaitNs : kWaitNs;
            while (ld_acquire_cta_shared(cnt) < target) {
                if (global_ns() - t0 > limit) {
                    atomicExch(p.status, SSD_ERR_TIMEOUT);
                    *broken = 1;
                    return;
                }
                __nanosleep(32);
            }
        };
        for (;;) {
            wait_bar(&bars.unit_full, par(ucnt), p.status, broken);
            ++ucnt;
            const int u = s_unit;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.unit_empty);
            if (u >= p.n_units) break;
            const Unit un = decode(u, p);
            if (!un.rows) continue;
            for (int h = un.h0 + pl; h < un.h1; h += 2) {
                const int bh = un.b * sh.H + h;
                if (un.owner) {
                    const bool writes = un.c < sh.nc - 1;
                    const bool publish = writes && !(bh == p.withhold_bh && un.c == p.withhold_c);
                    if (kD > 1 && writes) {
                        // L_c and sigma_c stored
                        wait_count(&s_agg[pl], kPipeWarps * ++acnt);
                        if (lane == 0 && publish) st_release_gpu(p.agg + bh * R + un.c % R, un.c + 1);
                    }
                    // the bf16 tile of S~_c (in the owner's W buffer) for the next chunk's other block goes to
                    // slot c % R once that slot's earlier readers are done (waited for while the owner's warps
                    // still work).  W is handed back (the drain stages y there) as soon as the store has read
                    // it, before inc is released (whose fence takes longer); tin is released once the store
                    // is complete.
                    const bool tile = kD == 1 && writes && p.halves == 2;
                    if (tile && lane == 0 && un.c >= R)
                        wait_flag(p.cons + bh * R + un.c % R, un.c / R, p.flag_polls, abort, p.status);
                    wait_count(&s_owned[pl], kPipeWarps * ++ocnt);
                    if (tile && lane == 0) {
                        tma_store_3d(&mR, sTile, 0, 0, bh * R + un.c % R);
                        bulk_commit();
                        bulk_wait_read();
                        mbar_arrive(&bars.pb[pl].t_free);
                    }
                    if (lane == 0 && publish) st_release_gpu(inc_flag<kD>(p.inc, bh, un.c), un.c + 1);
                    // with look-back the owner has read (at most) the slots of the D chunks before it:
                    // count them all (without, only owners read the fp32 state, each its one slot before
                    // the publication the next owner waits for)
                    if (kD > 1 && lane < min(kD, un.c)) red_release_add_gpu(p.cons + bh * R + (un.c - 1 - lane) % R, 1);
                    if (tile && lane == 0) {
                        bulk_wait_all();
                        fence_proxy_async_global();
                        if (publish) st_release_gpu(p.tin + bh * R + un.c % R, un.c + 1);
                    }
                } else if (un.c > 0) {
                    // the other block of chunk c has read S~_{c-1} (without look-back its issuer counts the tile
                    // once it landed, with look-back its eight warps their ring reads; chunk 0's block reads
                    // the initial state)
                    wait_count(&s_copied[pl], (kD == 1 ? 1 : kPipeWarps) * ++tcnt);
                    if (lane == 0) red_release_add_gpu(p.cons + bh * R + (un.c - 1) % R, 1);
                }
                __syncwarp();
            }
        }
    } else if (warp >= kSimtWarps) {
        // ------------------------------------------------------------------
        // Issuer warps: warp 16 drives pipeline 0 and also hands out units,
        // loads C and B and forms G; warp 17 drives pipeline 1.  The whole
        // warp follows the control flow and waits; lane 0 alone issues.
        // ------------------------------------------------------------------
        const int pl = warp - kSimtWarps;
        const bool leader = (lane == 0);
        PipeBars &pb = bars.pb[pl];
        uint8_t *sXlo = smem + kOffPipe + pl * kPipeBytes;
        uint8_t *sW = sXlo + 16384;
        uint8_t *sXhi = sXlo + 32768;
        const uint32_t tA = tmem + col_acc_a(pl), tB = tmem + col_acc_b(pl), tM = tmem + col_mask(pl);
        if (leader && pl == 0) {
            tma_prefetch_desc(&mC);
            tma_prefetch_desc(&mB);
            tma_prefetch_desc(&mX);
            tma_prefetch_desc(&mY);
        }
        const uint32_t idG = idesc_bf16_f32(kRows, kRows, 0, 0);    // C (K-major) x B (K-major)
        const uint32_t idState = idesc_bf16_f32(kRows, kP, 1, 1);   // B^T (MN-major) x scaled x (MN-major)
        const uint32_t idInter = idesc_bf16_f32(kRows, kP, 0, 1);   // C (K-major) x state tile [n][p]
        const uint32_t idMX = idesc_bf16_f32(kRows, kP, 0, 1);      // mask (TMEM) x x rows [i][p]
        uint32_t use = 0, ocnt = 0, ucnt = 0, cbcnt = 0, udone = 0;
        uint32_t scnt = 0, ecnt = 0;  // s_full and e_full phases (not every head has both)
        int next_u = -1;
        for (;;) {
            int u = 0;
            if (pl == 0) {
                if (ucnt > 0) wait_bar(&bars.unit_empty, par(ucnt - 1), p.status, broken);
                if (leader) {
                    u = (next_u >= 0) ? next_u : atomicAdd(p.counter, 1);
                    s_unit = u;
                    mbar_arrive(&bars.unit_full);
                }
                u = __shfl_sync(0xffffffffu, u, 0);
            } else {
                wait_bar(&bars.unit_full, par(ucnt), p.status, broken);
                u = s_unit;
                __syncwarp();
                if (leader) mbar_arrive(&bars.unit_empty);
            }
            ++ucnt;
            if (u >= p.n_units) break;
            const Unit un = decode(u, p);
            if (!un.rows) {
                next_u = -1;
                continue;
            }
            // this pipeline's first head of the unit: its x rows now, ahead of C, B and G (the pipeline's own
            // products of the previous unit have completed, so its x buffers are free)
            const int h_first = un.h0 + pl;
            if (leader && h_first < un.h1) {
                mbar_arrive_expect_tx(&pb.x_full, ((un.r == 1) ? 2u : 1u) * 16384u);
                tma_load_4d(sXlo, &mX, &pb.x_full, 0, h_first, un.t0, un.b);
                if (un.r == 1) tma_load_4d(sXhi, &mX, &pb.x_full, 0, h_first, un.t0 + kRows, un.b);
            }
            __syncwarp();
            if (pl == 0) {
                // both pipelines are done with the previous unit's C, B and G
                if (udone > 0) wait_bar(&bars.unit_done, par(udone - 1), p.status, broken);
                if (leader) {
                    const uint32_t bboxes = (un.r == 1) ? 2u : 1u;
                    mbar_arrive_expect_tx(&bars.cb, (uint32_t)(NK + 2 * bboxes) * 16384u);
                    for (int k = 0; k < NK; ++k)
                        tma_load_4d(sC + k * 16384, &mC, &bars.cb, k * 64, un.g, un.t0 + un.row0, un.b);
                    for (int k = 0; k < 2; ++k)
                        for (uint32_t q = 0; q < bboxes; ++q)
                            tma_load_4d(sB + k * 32768 + q * 16384, &mB, &bars.cb, k * 64, un.g,
                                        un.t0 + (int)q * kRows, un.b);
                    // claim the next unit now and warm L2 with its first tiles
                    next_u = atomicAdd(p.counter, 1);
                    if (next_u < p.n_units) {
                        const Unit nx = decode(next_u, p);
                        if (nx.rows) {
                            for (int k = 0; k < NK; ++k)
                                tma_prefetch_4d(&mC, k * 64, nx.g, nx.t0 + nx.row0, nx.b);
                            for (int k = 0; k < 2; ++k)
                                for (int q = 0; q <= nx.r; ++q)
                                    tma_prefetch_4d(&mB, k * 64, nx.g, nx.t0 + q * kRows, nx.b);
                            for (int hh = nx.h0; hh < min(nx.h0 + 2, nx.h1); ++hh)
                                for (int q = 0; q <= nx.r; ++q)
                                    tma_prefetch_4d(&mX, 0, hh, nx.t0 + q * kRows, nx.b);
                            // the chunk's dt (all heads: one contiguous block) for the first prefix sums
                            const float *dtb = p.dt + ((size_t)nx.b * sh.T + nx.t0) * sh.H;
                            const uint32_t dtbytes = ((uint32_t)nx.len * sh.H * 4u) & ~15u;
                            if ((reinterpret_cast<uintptr_t>(dtb) & 15) == 0 && dtbytes > 0)
                                bulk_prefetch_l2(dtb, dtbytes);
                        }
                    }
                }
                next_u = __shfl_sync(0xffffffffu, next_u, 0);
            }
            ++udone;
            wait_bar(&bars.cb, par(cbcnt++), p.status, broken);
            fence_after_sync();
            if (pl == 0) {
                // G = C_r B_r^T: the block's rows against its own columns, K = N
                if (leader) {
                    for (int kk = 0; kk < NK * 4; ++kk) {
                        const int atom = kk >> 2, kin = kk & 3;
                        mma_ss(tmem + kColG,
                               smem_desc_sw128(smem_u32(sC) + atom * 16384 + kin * 32, 16, 1024),
                               smem_desc_sw128(smem_u32(sB) + atom * 32768 + un.row0 * 128 + kin * 32, 16, 1024),
                               idG, kk > 0);
                    }
                    mma_commit(&bars.g_done);
                }
                __syncwarp();
            }
            // x rows of this block; the entering-state tile: for an owner of the second block x rows
            // 0..127 (free once its state products are done; W then holds its bf16 tile of S~_c), W for
            // the only block, the unused x buffer for another block (so that it need not wait for the
            // previous head's y tile to leave W)
            uint8_t *sXr = (un.r == 1) ? sXhi : sXlo;
            uint8_t *sE = un.owner ? (un.r == 1 ? sXlo : sW) : sXhi;
            bool any = false;
            for (int h = un.h0 + pl; h < un.h1; h += 2, ++use) {
                any = true;
                // this head's x rows (the unit's first head's are already on their way); warm L2 for the
                // pipeline's next head
                if (use > 0) wait_bar(&pb.mx_done, par(use - 1), p.status, broken);
                if (leader) {
                    const uint32_t xboxes = (un.r == 1) ? 2u : 1u;
                    if (h != h_first) {
                        mbar_arrive_expect_tx(&pb.x_full, xboxes * 16384u);
                        tma_load_4d(sXlo, &mX, &pb.x_full, 0, h, un.t0, un.b);
                        if (un.r == 1) tma_load_4d(sXhi, &mX, &pb.x_full, 0, h, un.t0 + kRows, un.b);
                    }
                    if (h + 2 < un.h1)
                        for (uint32_t q = 0; q < xboxes; ++q)
                            tma_prefetch_4d(&mX, 0, h + 2, un.t0 + (int)q * kRows, un.b);
                }
                __syncwarp();
                // without look-back another block past chunk 0 takes S~_{c-1} as the bf16 tile its owner
                // stored: loaded here once published (while the CUDA-core warps build the mask), counted as
                // read once it landed
                const bool e_tma = kD == 1 && !un.owner && un.c > 0;
                if (e_tma) {
                    if (leader) {
                        const int bh = un.b * sh.H + h;
                        wait_flag(p.tin + bh * R + (un.c - 1) % R, un.c, p.flag_polls, abort, p.status);
                        if (!*abort) {
                            fence_proxy_async_global();
                            mbar_arrive_expect_tx(&pb.e_full, (uint32_t)p.tile_rows * 128u);
                            tma_load_3d(sXhi, &mR, &pb.e_full, 0, 0, bh * R + (un.c - 1) % R);
                        } else {
                            mbar_arrive(&pb.e_full);  // given up: no copy, the phase completes at once
                        }
                    }
                    __syncwarp();
                }
                if (un.owner) {
                    // stages 2-3 products: S_pre = B_{<r}^T (scaled rows before the block) into A,
                    // S_own = B_r^T (scaled rows of the block) into B; M = n, N = p, K = tokens
                    wait_bar(&pb.x_full, par(use), p.status, broken);
                    wait_bar(&pb.xd_full, par(ocnt), p.status, broken);
                    if (use > 0) wait_bar(&pb.acc_free, par(use - 1), p.status, broken);
                    fence_after_sync();
                    if (leader) {
                        if (un.r == 1)
                            for (int kk = 0; kk < 8; ++kk)
                                mma_ss(tA, smem_desc_sw128(smem_u32(sB) + kk * 2048, 32768, 1024),
                                       smem_desc_sw128(smem_u32(sXlo) + kk * 2048, 16, 1024), idState, kk > 0);
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ss(tB, smem_desc_sw128(smem_u32(sB) + un.row0 * 128 + kk * 2048, 32768, 1024),
                                   smem_desc_sw128(smem_u32(sW) + kk * 2048, 16, 1024), idState, kk > 0);
                        mma_commit(&pb.d_done);
                    }
                    __syncwarp();
                    ++ocnt;
                }
                // stage 4 product: Y_inter = C_r E^T into A (E: the entering-state tile [n][p])
                if (e_tma) {
                    wait_bar(&pb.e_full, par(ecnt++), p.status, broken);
                    if (leader && un.c > 0) red_release_cta_shared_add(&s_copied[pl], 1);
                } else {
                    wait_bar(&pb.s_full, par(scnt++), p.status, broken);
                }
                if (!un.owner && use > 0) wait_bar(&pb.acc_free, par(use - 1), p.status, broken);
                fence_after_sync();
                if (leader) {
                    for (int kk = 0; kk < NK * 4; ++kk) {
                        const int atom = kk >> 2, kin = kk & 3;
                        mma_ss(tA, smem_desc_sw128(smem_u32(sC) + atom * 16384 + kin * 32, 16, 1024),
                               smem_desc_sw128(smem_u32(sE) + kk * 2048, 16, 1024), idInter, kk > 0);
                    }
                }
                __syncwarp();
                // stage 1 product: Y_intra = M X_r into B
                wait_bar(&pb.m_full, par(use), p.status, broken);
                if (!un.owner) wait_bar(&pb.x_full, par(use), p.status, broken);
                fence_after_sync();
                if (leader) {
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ts(tB, tM + kk * 8, smem_desc_sw128(smem_u32(sXr) + kk * 2048, 16, 1024), idMX,
                               kk > 0);
                    mma_commit(&pb.mx_done);
                }
                __syncwarp();
            }
            // this pipeline is done with the unit once its last products completed
            if (any) wait_bar(&pb.mx_done, par(use - 1), p.status, broken);
            if (leader) mbar_arrive(&bars.unit_done);
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------------
        // CUDA-core warps: warps 8pl..8pl+7 serve pipeline pl.  Thread wtid
        // owns token wtid of the chunk for the prefix sums; for tile work,
        // warp quarter q (warp & 3) owns TMEM lanes 32q..32q+31 (rows of
        // the block, or n of a state) and warpgroup `half` owns columns
        // 32 half .. 32 half + 31 of every 64-wide tile.  One thread (`ctl`,
        // the first of warpgroup 1, whose warp has the least mask work) waits
        // on other CTAs' flags and issues the y stores.
        // ------------------------------------------------------------------
        const int pl = warp >> 3;
        const int pw = warp & 7;
        const int half = pw >> 2;
        const int quarter = warp & 3;
        const int wtid = pw * 32 + lane;
        const bool ctl = (wtid == kPipeThreads / 2);
        const int lrow = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const int bar_id = 1 + pl;       // the pipeline's 256 threads
        const int bar_wg1 = 3 + pl;      // its second warpgroup (the one holding ctl)
        PipeBars &pb = bars.pb[pl];
        uint8_t *sXlo = smem + kOffPipe + pl * kPipeBytes;
        uint8_t *sW = sXlo + 16384;
        uint8_t *sXhi = sXlo + 32768;
        float *sJ = reinterpret_cast<float *>(smem + kOffAux) + pl * kAuxFloats;  // s in log2 units
        float *sF = sJ + 256;                                                     // column factors
        float *sTot = sF + 256;                                                   // warp totals
        float *sWB = reinterpret_cast<float *>(smem + kOffWB) + pl * 2 * kP;      // gated: weight, bias
        const uint32_t tA = tmem + col_acc_a(pl), tB = tmem + col_acc_b(pl), tM = tmem + col_mask(pl);
        const size_t PN = (size_t)kP * N;
        uint32_t use = 0, ocnt = 0, ucnt = 0, gcnt = 0, tcnt = 0;  // tcnt: this pipeline's stored state tiles

        // stage 0: inclusive prefix sums of dt*A over the chunk, in log2 units, into sJ (and the
        // mask's column factors exp(s_{i|31} - s_i) <= 1 into sF); every thread of the pipeline
        auto scan = [&](float dtv, float a) {
            float v = dtv * (a * kLog2e);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float t = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += t;
            }
            if (lane == 31) sTot[pw] = v;
            named_bar_sync(bar_id, kPipeThreads);
            float pre = 0.f;
            for (int w = 0; w < pw; ++w) pre += sTot[w];
            const float s_mine = pre + v;
            sJ[wtid] = s_mine;
            sF[wtid] = ex2(__shfl_sync(0xffffffffu, s_mine, 31) - s_mine);
            named_bar_sync(bar_id, kPipeThreads);
        };
        for (;;) {
            wait_bar(&bars.unit_full, par(ucnt), p.status, broken);
            ++ucnt;
            const int u = s_unit;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.unit_empty);
            if (u >= p.n_units) break;
            const Unit un = decode(u, p);
            if (!un.rows) continue;
            const uint32_t gphase = gcnt++;
            int h = un.h0 + pl;
            if (h >= un.h1) continue;
            const bool own = un.owner;
            const int end = un.len - 1;
            const int j = un.row0 + lrow;  // this thread's row of the chunk
            const float *dtp = p.dt + ((size_t)un.b * sh.T + un.t0 + wtid) * sh.H;
            float dt_next = 0.f, a_next = 0.f, d_cur = p.D ? __ldg(p.D + h) : 0.f;
            scan((wtid < un.len) ? __ldg(dtp + h) : 0.f, __ldg(p.A + h));
            // an owner's ctl reads `inc` of the chunk before for the pipeline's head early (acquire), so
            // that the wait usually costs nothing by the time the state is needed (ctl's warp builds only
            // zero mask slabs); another block's issuer waits for it instead
            int ready_seen = (ctl && (own || kD > 1) && un.c > 0)
                                 ? ld_acquire_gpu(inc_flag<kD>(p.inc, un.b * sh.H + h, un.c - 1))
                                 : 0;
            bool first_head = true;
            for (; h < un.h1; h += 2, ++use) {
                const int bh = un.b * sh.H + h;
                const bool has_next = h + 2 < un.h1;
                // the next head's dt, A and D, in flight while this head is processed
                if (has_next) {
                    dt_next = (wtid < un.len) ? __ldg(dtp + h + 2) : 0.f;
                    a_next = __ldg(p.A + h + 2);
                }
                const float Dh = d_cur;
                if (has_next) d_cur = p.D ? __ldg(p.D + h + 2) : 0.f;
                // gated drain: this head's z rows on their way to L2 (one 128-byte line per row), and its norm
                // weight and bias into shared memory (an async copy: no register, so no barrier waits for it)
                if (kGated) {
                    if (half == 0 && j < un.len) prefetch_l2(p.z + (((size_t)un.b * sh.T + un.t0 + j) * sh.H + h) * kP);
                    if (wtid < 32) {
                        const float *src = (wtid < 16) ? p.gw : p.gb;
                        if (src) cp_async16(sWB + wtid * 4, src + h * kP + (wtid & 15) * 4);
                    }
                }
                const float s_end = sJ[end];
                const float s_ref = (un.r == 1) ? sJ[kRows - 1] : 0.f;  // s_{r-1}
                const float sj = sJ[j];
                const float ej = ex2(sj - s_ref);
                const bool writes_ring = own && un.c < sh.nc - 1;

                // ---- owner: rows scaled by their decay to the state's end (stage 2 operand)
                if (own) {
                    wait_bar(&pb.x_full, par(use), p.status, broken);
                    if (un.r == 1) {
                        // rows 0..127 in place (to row 127: S_pre, warpgroup 0), rows 128..255 into W
                        // (to the end, warpgroup 1, once the previous y tile has left W)
                        const int row = wtid;
                        const bool lo = row < kRows;
                        if (!lo) {
                            if (ctl) bulk_wait_read();
                            named_bar_sync(bar_wg1, kPipeThreads / 2);
                        }
                        const float w = ex2((lo ? s_ref : s_end) - sJ[row]);
                        const uint8_t *src = (lo ? sXlo : sXhi);
                        uint8_t *dst = lo ? sXlo : sW;
                        const int rr = row & (kRows - 1);
                        uint4 xv[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) xv[k] = lds128(src + swz(rr, k));
#pragma unroll
                        for (int k = 0; k < 8; ++k) sts128(dst + swz(rr, k), scale_bf16x8(xv[k], w));
                    } else {
                        // the only block: rows 0..127 into W (to the end); x stays unscaled for M X
                        if (ctl) bulk_wait_read();
                        named_bar_sync(bar_id, kPipeThreads);
                        const int rr = wtid & (kRows - 1), k0 = (wtid >> 7) * 4;
                        const float w = ex2(s_end - sJ[rr]);
                        uint4 xv[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) xv[k] = lds128(sXlo + swz(rr, k0 + k));
#pragma unroll
                        for (int k = 0; k < 4; ++k) sts128(sW + swz(rr, k0 + k), scale_bf16x8(xv[k], w));
                    }
                    fence_view_async_shared();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pb.xd_full);
                }

                // ---- stage 1 mask M[j][i] = exp(s_j - s_i) G[j][i] for i <= j (+ D_h at i = j), bf16 in
                // TMEM, in 32-column slabs: below the diagonal slab a row factor times a column factor
                // (both <= 1), in it one exponential per element (about three times the work), above
                // it zeros.  Warpgroup 0 takes the diagonal slab, warpgroup 1 the other three.
                // an owner's slot count, read (acquire) before the mask for the same reason
                int cons_seen = 0;
                if (kD > 1 && own && ctl && writes_ring && un.c >= R)
                    cons_seen = ld_acquire_gpu(p.cons + bh * R + un.c % R);
                if (first_head) wait_bar(&bars.g_done, par(gphase), p.status, broken);
                fence_after_sync();
                {
                    const int dq = quarter;  // diagonal slab of this warp's rows
#pragma unroll 1
                    for (int sl = 0; sl < 4; ++sl) {
                        const bool mine = (half == 0) ? (sl == dq) : (sl != dq);
                        if (!mine) continue;
                        uint32_t o[16];
                        if (sl > dq) {
#pragma unroll
                            for (int q = 0; q < 16; ++q) o[q] = 0u;
                        } else {
                            uint32_t g[32];
                            tmem_ld16(tmem + kColG + sl * 32 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&g[0]));
                            tmem_ld16(tmem + kColG + sl * 32 + 16 + lane_base,
                                      *reinterpret_cast<uint32_t(*)[16]>(&g[16]));
                            tmem_wait_ld();
                            if (sl == dq) {
                                const float2 *sc = reinterpret_cast<const float2 *>(sJ + un.row0 + dq * 32);
#pragma unroll
                                for (int q = 0; q < 16; ++q) {
                                    const float2 si = sc[q];
                                    float a = (2 * q <= lane) ? __uint_as_float(g[2 * q]) * ex2(sj - si.x) : 0.f;
                                    float b =
                                        (2 * q + 1 <= lane) ? __uint_as_float(g[2 * q + 1]) * ex2(sj - si.y) : 0.f;
                                    if (2 * q == lane) a += Dh;
                                    if (2 * q + 1 == lane) b += Dh;
                                    o[q] = pack_bf16x2(a, b);
                                }
                            } else {
                                const int i0 = un.row0 + sl * 32;
                                const float rf = ex2(sj - sJ[i0 + 31]);
                                const float2 rr = make_float2(rf, rf);
                                const float4 *f4 = reinterpret_cast<const float4 *>(sF + i0);
#pragma unroll
                                for (int q = 0; q < 8; ++q) {
                                    const float4 f = f4[q];
                                    const float2 w0 = mul_f32x2(rr, make_float2(f.x, f.y));
                                    const float2 w1 = mul_f32x2(rr, make_float2(f.z, f.w));
                                    const float2 m0 = mul_f32x2(
                                        make_float2(__uint_as_float(g[4 * q]), __uint_as_float(g[4 * q + 1])), w0);
                                    const float2 m1 = mul_f32x2(
                                        make_float2(__uint_as_float(g[4 * q + 2]), __uint_as_float(g[4 * q + 3])),
                                        w1);
                                    o[2 * q] = pack_bf16x2(m0.x, m0.y);
                                    o[2 * q + 1] = pack_bf16x2(m1.x, m1.y);
                                }
                            }
                        }
                        tmem_st16(tM + sl * 16 + lane_base, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
                    }
                    tmem_wait_st();
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pb.m_full);
                }
                first_head = false;
                // the previous y tile has left W before any thread writes W again (the next barrier of
                // the pipeline publishes this)
                if (ctl) bulk_wait_read();

                // ---- stage 3: the state entering the block
                // An owner's bf16 tile of S~_c, for the next chunk's other block: row n of the 128-byte-swizzled
                // [n][p] tile in W (free once the state products are done; the drain waits for the store
                // before it stages y there), rows past N zero; the publisher stores it with TMA.
                const int n = lrow;  // state row of this thread (TMEM lane); p in [32 half, 32 half + 32)
                const bool nv = n < N;
                auto store_tile = [&](const float (&v)[32]) {
                    if (n < p.tile_rows) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            uint4 t;
                            t.x = pack_bf16x2(v[8 * k + 0], v[8 * k + 1]);
                            t.y = pack_bf16x2(v[8 * k + 2], v[8 * k + 3]);
                            t.z = pack_bf16x2(v[8 * k + 4], v[8 * k + 5]);
                            t.w = pack_bf16x2(v[8 * k + 6], v[8 * k + 7]);
                            if (!nv) t = make_uint4(0u, 0u, 0u, 0u);
                            sts128(sW + swz(n, half * 4 + k), t);
                        }
                    }
                    fence_view_async_shared();
                };
                if (kD == 1 && !own && un.c > 0) {
                    // another block past chunk 0: its issuer loads the entering state, the bf16 tile of
                    // S~_{c-1}, by TMA.  Without the next head's prefix sums below, this barrier is the one
                    // that orders ctl's wait for the previous y tile before the drain writes W.
                    if (!has_next) named_bar_sync(bar_id, kPipeThreads);
                } else if constexpr (kD == 1) {
                    // without look-back: an owner takes S~_{c-1} (published by the owner of chunk c-1) from
                    // the sequence's one fp32 slot and writes S~_c over it (the next owner, the slot's only
                    // other reader, waits for this one's publication); chunk 0's blocks take the initial
                    // state.  The bf16 tile of S~_c goes to slot c % 3 of the tile ring, which held chunk
                    // c-3's, read by the other block of chunk c-2; the publisher waits for that read (the
                    // other blocks of chunks k >= 1 read slot (k - 1) % 3, so the slot has had c / 3 counted
                    // reads once that one is in).
                    if (ctl && un.c > 0 && ready_seen < un.c)
                        wait_flag(inc_flag<kD>(p.inc, bh, un.c - 1), un.c, p.flag_polls, abort, p.status);
                    named_bar_sync(bar_id, kPipeThreads);
                    float old[32];
                    if (un.c == 0) {
                        const size_t ld = p.state_ld;
                        const int pv = p.p_full - p.p_off - half * 32;  // valid state rows among this thread's 32
                        const float *src =
                            p.init ? p.init + ((size_t)bh * p.p_full + p.p_off + half * 32) * ld + p.n_off + n : nullptr;
#pragma unroll
                        for (int q = 0; q < 32; ++q) old[q] = (src && nv && q < pv) ? __ldg(src + (size_t)q * ld) : 0.f;
                    } else {
                        const float4 *src = reinterpret_cast<const float4 *>(p.ring + (size_t)bh * PN);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 t =
                                nv ? __ldcg(src + ring_quad(N, n, half * 8 + q)) : make_float4(0.f, 0.f, 0.f, 0.f);
                            old[4 * q] = t.x;
                            old[4 * q + 1] = t.y;
                            old[4 * q + 2] = t.z;
                            old[4 * q + 3] = t.w;
                        }
                    }
                    // the entering-state tile [n][p], B operand of stage 4 (as the issuer's sE)
                    uint8_t *sE = own ? (un.r == 1 ? sXlo : sW) : sXhi;
                    if (own) {
                        wait_bar(&pb.d_done, par(ocnt), p.status, broken);
                        ++ocnt;
                        fence_after_sync();
                        if (un.r == 1) {
                            // E = exp(s_127) S~_{c-1} + S_pre
                            const float e_start = ex2(s_ref);
#pragma unroll
                            for (int q0 = 0; q0 < 32; q0 += 16) {
                                uint32_t t[16];
                                tmem_ld16(tA + half * 32 + q0 + lane_base, t);
                                tmem_wait_ld();
#pragma unroll
                                for (int q = 0; q < 16; ++q)
                                    old[q0 + q] = fmaf(e_start, old[q0 + q], __uint_as_float(t[q]));
                            }
                        }
                    }
                    // E in bf16 into row n of the tile (128-byte swizzled)
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint4 t;
                        t.x = pack_bf16x2(old[8 * k + 0], old[8 * k + 1]);
                        t.y = pack_bf16x2(old[8 * k + 2], old[8 * k + 3]);
                        t.z = pack_bf16x2(old[8 * k + 4], old[8 * k + 5]);
                        t.w = pack_bf16x2(old[8 * k + 6], old[8 * k + 7]);
                        if (!nv) t = make_uint4(0u, 0u, 0u, 0u);
                        sts128(sE + swz(n, half * 4 + k), t);
                    }
                    fence_view_async_shared();
                    if (!own) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&pb.s_full);  // chunk 0's other block: the initial state
                    } else {
                        // S~_c = exp(s_end - s_{r-1}) E + S_own.  S_own is read from TMEM before s_full,
                        // after which the issuer overwrites that accumulator.
                        const float e_rest = ex2(s_end - s_ref);
#pragma unroll
                        for (int q0 = 0; q0 < 32; q0 += 16) {
                            uint32_t t[16];
                            tmem_ld16(tB + half * 32 + q0 + lane_base, t);
                            tmem_wait_ld();
#pragma unroll
                            for (int q = 0; q < 16; ++q) old[q0 + q] = fmaf(e_rest, old[q0 + q], __uint_as_float(t[q]));
                        }
                        fence_before_sync();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&pb.s_full);
                        if (writes_ring) {
                            float4 *dst = reinterpret_cast<float4 *>(p.ring + (size_t)bh * PN);
                            if (nv) {
#pragma unroll
                                for (int q = 0; q < 8; ++q)
                                    __stcg(dst + ring_quad(N, n, half * 8 + q),
                                           make_float4(old[4 * q], old[4 * q + 1], old[4 * q + 2], old[4 * q + 3]));
                            }
                            if (p.halves == 2) store_tile(old);
                        } else if (nv && p.fin) {
                            const size_t ld = p.state_ld;
                            const int pv = p.p_full - p.p_off - half * 32;
                            float *fin = p.fin + ((size_t)bh * p.p_full + p.p_off + half * 32) * ld + p.n_off + n;
#pragma unroll
                            for (int q = 0; q < 32; ++q)
                                if (q < pv) fin[(size_t)q * ld] = old[q];
                        }
                        __syncwarp();
                        if (lane == 0) red_release_cta_shared_add(&s_owned[pl], 1);  // the publisher releases the stores
                    }
                } else {
                    // look-back: the owner may start from an earlier S~_j and fold in the local states
                    // after it, S~_i = exp(sigma_i) S~_{i-1} + L_i.  Every owner forms its own S~_c by
                    // that same fp32 expression, so the result does not depend on where the fold
                    // started.  Chunk c's states go to slot c % R, which held chunk c - R's: the owner
                    // overwrites it once that chunk's readers (the D owners after it and the next
                    // chunk's other block) have all added themselves to `cons`.
                    const int reads_per_use = kD + (p.halves == 2 ? 1 : 0);
                    const size_t PN2 = 2 * PN;  // a slot: S~, then L
                    const float *ring_bh = p.ring + (size_t)bh * R * PN2;
                    const int quad0 = half * 8;
                    if (own && writes_ring) {
                        // publish L_c = exp(s_end - s_{r-1}) S_pre + S_own (S_own alone for r = 0) and
                        // sigma_c as soon as the state products are done
                        if (ctl && un.c >= R && cons_seen < (un.c / R) * reads_per_use)
                            wait_flag(p.cons + bh * R + un.c % R, (un.c / R) * reads_per_use, p.flag_polls, abort,
                                      p.status);
                        named_bar_sync(bar_id, kPipeThreads);
                    }
                    if (own) {
                        wait_bar(&pb.d_done, par(ocnt), p.status, broken);
                        ++ocnt;
                        fence_after_sync();
                    }
                    if (own && writes_ring) {
                        const float e_rest = ex2(s_end - s_ref);
                        float4 *dst = reinterpret_cast<float4 *>(const_cast<float *>(ring_bh) + (un.c % R) * PN2 + PN);
#pragma unroll
                        for (int q0 = 0; q0 < 32; q0 += 8) {
                            uint32_t a[8], b[8];
                            if (un.r == 1) tmem_ld8(tA + half * 32 + q0 + lane_base, a);
                            tmem_ld8(tB + half * 32 + q0 + lane_base, b);
                            tmem_wait_ld();
                            float l[8];
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                l[q] = (un.r == 1) ? fmaf(e_rest, __uint_as_float(a[q]), __uint_as_float(b[q]))
                                                   : __uint_as_float(b[q]);
                            if (nv) {
                                __stcg(dst + ring_quad(N, n, quad0 + q0 / 4), make_float4(l[0], l[1], l[2], l[3]));
                                __stcg(dst + ring_quad(N, n, quad0 + q0 / 4 + 1), make_float4(l[4], l[5], l[6], l[7]));
                            }
                        }
                        if (ctl) __stcg(p.sig + bh * R + un.c % R, s_end);
                        __syncwarp();
                        if (lane == 0) red_release_cta_shared_add(&s_agg[pl], 1);  // the publisher releases them
                    }
                    int base = un.c - 1;  // the chunk whose S~ the fold starts from (-1: the initial state)
                    if (own) {
                        // ctl's warp polls the flags of the D chunks before this one at once (lane l:
                        // chunk c-1-l) and takes the most recent S~_j whose later chunks all have L out
                        if ((wtid >> 5) == 4) {
                            const unsigned full = 0xffffffffu;
                            const int jl = un.c - 1 - lane;
                            const bool seen = __shfl_sync(full, ready_seen, 0) >= un.c;  // S~_{c-1} seen early
                            uint32_t polls = 0;
                            int found = seen ? un.c - 1 : -2;
                            while (found == -2) {
                                bool inc_ok = false, agg_ok = false;
                                if (lane < kD) {
                                    if (jl >= 0) {
                                        inc_ok = ld_acquire_gpu(inc_flag<kD>(p.inc, bh, jl)) >= jl + 1;
                                        agg_ok = ld_acquire_gpu(p.agg + bh * R + jl % R) >= jl + 1;
                                    } else {
                                        inc_ok = (jl == -1);  // the initial state
                                    }
                                }
                                const unsigned im = __ballot_sync(full, inc_ok), am = __ballot_sync(full, agg_ok);
                                const int run = __ffs(~am) - 1;  // chunks c-1 .. c-run have L published
                                const unsigned cand = im & ((2u << run) - 1u);
                                if (cand) {
                                    found = un.c - __ffs(cand);
                                    break;
                                }
                                bool give_up = *abort != 0;
                                if (!give_up && ++polls >= p.flag_polls) {
                                    if (lane == 0) atomicExch(p.status, SSD_ERR_TIMEOUT);
                                    give_up = true;
                                }
                                if (!give_up && ld_relaxed_gpu(p.status) != 0) give_up = true;
                                if (__any_sync(full, give_up)) {
                                    if (lane == 0) *abort = 1;
                                    found = max(un.c - kD, -1);  // in bounds; the results are not valid
                                    break;
                                }
                                __nanosleep(64);
                            }
                            __syncwarp();
                            if (lane == 0) s_base[pl] = found;
                        }
                        named_bar_sync(bar_id, kPipeThreads);
                        base = s_base[pl];
                    } else {
                        // another block reads S~_{c-1} from the ring (chunk 0's the initial state)
                        if (ctl && un.c > 0 && ready_seen < un.c)
                            wait_flag(inc_flag<kD>(p.inc, bh, un.c - 1), un.c, p.flag_polls, abort, p.status);
                        named_bar_sync(bar_id, kPipeThreads);
                    }
                    float old[32];
                    if (base < 0) {
                        const size_t ld = p.state_ld;
                        const int pv = p.p_full - p.p_off - half * 32;  // valid state rows among this thread's 32
                        const float *src =
                            p.init ? p.init + ((size_t)bh * p.p_full + p.p_off + half * 32) * ld + p.n_off + n : nullptr;
#pragma unroll
                        for (int q = 0; q < 32; ++q) old[q] = (src && nv && q < pv) ? __ldg(src + (size_t)q * ld) : 0.f;
                    } else {
                        const float4 *src = reinterpret_cast<const float4 *>(ring_bh + (base % R) * PN2);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 t = nv ? __ldcg(src + ring_quad(N, n, quad0 + q)) : make_float4(0.f, 0.f, 0.f, 0.f);
                            old[4 * q] = t.x;
                            old[4 * q + 1] = t.y;
                            old[4 * q + 2] = t.z;
                            old[4 * q + 3] = t.w;
                        }
                    }
#pragma unroll 1
                    for (int i = base + 1; i < un.c; ++i) {
                        const float e = ex2(__ldcg(p.sig + bh * R + i % R));
                        const float4 *src = reinterpret_cast<const float4 *>(ring_bh + (i % R) * PN2 + PN);
                        float4 t[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            t[q] = nv ? __ldcg(src + ring_quad(N, n, quad0 + q)) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            old[4 * q] = fmaf(e, old[4 * q], t[q].x);
                            old[4 * q + 1] = fmaf(e, old[4 * q + 1], t[q].y);
                            old[4 * q + 2] = fmaf(e, old[4 * q + 2], t[q].z);
                            old[4 * q + 3] = fmaf(e, old[4 * q + 3], t[q].w);
                        }
                    }
                    // the entering-state tile [n][p], B operand of stage 4 (as the issuer's sE)
                    uint8_t *sE = own ? (un.r == 1 ? sXlo : sW) : sXhi;
                    if (own) {
                        // E = exp(s_{r-1}) S~_{c-1} + S_pre (S~_{c-1} for r = 0) into the tile, and
                        // S~_c = exp(sigma_c) S~_{c-1} + L_c in place, with L_c exactly as published.  S_pre
                        // and S_own are read from TMEM before s_full, after which the issuer overwrites them.
                        const float e_start = ex2(s_ref), e_rest = ex2(s_end - s_ref), e_c = ex2(s_end);
#pragma unroll
                        for (int q0 = 0; q0 < 32; q0 += 8) {
                            uint32_t a[8], b[8];
                            if (un.r == 1) tmem_ld8(tA + half * 32 + q0 + lane_base, a);
                            tmem_ld8(tB + half * 32 + q0 + lane_base, b);
                            tmem_wait_ld();
                            uint32_t e[4];
#pragma unroll
                            for (int q = 0; q < 8; q += 2) {
                                float ev[2];
#pragma unroll
                                for (int k = 0; k < 2; ++k) {
                                    const float o = old[q0 + q + k];
                                    const float sp = (un.r == 1) ? __uint_as_float(a[q + k]) : 0.f;
                                    const float so = __uint_as_float(b[q + k]);
                                    ev[k] = (un.r == 1) ? fmaf(e_start, o, sp) : o;
                                    const float l = (un.r == 1) ? fmaf(e_rest, sp, so) : so;
                                    old[q0 + q + k] = fmaf(e_c, o, l);
                                }
                                e[q / 2] = pack_bf16x2(ev[0], ev[1]);
                            }
                            sts128(sE + swz(n, half * 4 + q0 / 8),
                                   nv ? make_uint4(e[0], e[1], e[2], e[3]) : make_uint4(0u, 0u, 0u, 0u));
                        }
                        fence_view_async_shared();
                        fence_before_sync();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&pb.s_full);
                        if (writes_ring) {
                            float4 *dst = reinterpret_cast<float4 *>(const_cast<float *>(ring_bh) + (un.c % R) * PN2);
                            if (nv) {
#pragma unroll
                                for (int q = 0; q < 8; ++q)
                                    __stcg(dst + ring_quad(N, n, quad0 + q),
                                           make_float4(old[4 * q], old[4 * q + 1], old[4 * q + 2], old[4 * q + 3]));
                            }
                        } else if (nv && p.fin) {
                            const size_t ld = p.state_ld;
                            const int pv = p.p_full - p.p_off - half * 32;
                            float *fin = p.fin + ((size_t)bh * p.p_full + p.p_off + half * 32) * ld + p.n_off + n;
#pragma unroll
                            for (int q = 0; q < 32; ++q)
                                if (q < pv) fin[(size_t)q * ld] = old[q];
                        }
                        __syncwarp();
                        if (lane == 0) red_release_cta_shared_add(&s_owned[pl], 1);  // the publisher releases the stores
                    } else {
                        // S~_{c-1} (or the initial state) in bf16 into row n of the tile
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            uint4 t;
                            t.x = pack_bf16x2(old[8 * k + 0], old[8 * k + 1]);
                            t.y = pack_bf16x2(old[8 * k + 2], old[8 * k + 3]);
                            t.z = pack_bf16x2(old[8 * k + 4], old[8 * k + 5]);
                            t.w = pack_bf16x2(old[8 * k + 6], old[8 * k + 7]);
                            if (!nv) t = make_uint4(0u, 0u, 0u, 0u);
                            sts128(sE + swz(n, half * 4 + k), t);
                        }
                        fence_view_async_shared();
                        __syncwarp();
                        if (lane == 0) {
                            mbar_arrive(&pb.s_full);
                            // the ring entries are consumed: the publisher may count the slot as read
                            if (un.c > 0) red_release_cta_shared_add(&s_copied[pl], 1);
                        }
                    }
                }

                // the next head's prefix sums, while this head's products run
                if (has_next) scan(dt_next, a_next);

                // gated drain: z of this row's 32 channels (in L2 since the head's start), loaded after the
                // prefix sums, whose barriers would otherwise wait for these loads
                uint4 zv[4];
                if (kGated) {
                    const bool jv = j < un.len;
                    const uint4 *zp = reinterpret_cast<const uint4 *>(
                        p.z + (((size_t)un.b * sh.T + un.t0 + j) * sh.H + h) * kP + half * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q) zv[q] = jv ? __ldg(zp + q) : make_uint4(0u, 0u, 0u, 0u);
                }


                // ---- stages 4-5: y_j = exp(s_j - s_{r-1}) Y_inter + Y_intra (the D skip is in the mask),
                // staged as bf16 in W (128-byte swizzled [j][p]) and written by one TMA store (rows
                // past T are clipped).  The second half of a 256-wide state adds the first half's y.
                uint4 yprev[4];
                if (kAccum) {
                    const bool jv = j < un.len;
                    const int pv = p.p_full - p.p_off - half * 32;
                    const uint4 *yp = reinterpret_cast<const uint4 *>(  // p.y starts at column p_off
                        p.y + (((size_t)un.b * sh.T + un.t0 + j) * sh.H + h) * p.p_full + half * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        yprev[q] = (jv && 8 * q < pv) ? __ldg(yp + q) : make_uint4(0u, 0u, 0u, 0u);
                }
                wait_bar(&pb.mx_done, par(use), p.status, broken);
                // an owner's bf16 state tile is in W until the publisher's store has read it
                if (kD == 1 && writes_ring && p.halves == 2) wait_bar(&pb.t_free, par(tcnt++), p.status, broken);
                fence_after_sync();
                if constexpr (kGated) {
                    // g = y * silu(z) in fp32 (y is never rounded), then the row's 64 channels normalised:
                    // two passes over this thread's 32, merged with the other warpgroup's through shared
                    // memory (mean and sum of squared deviations of two halves of 32)
                    float g[32];
#pragma unroll
                    for (int q0 = 0; q0 < 32; q0 += 16) {
                        uint32_t a[16], b[16];
                        tmem_ld16(tA + half * 32 + q0 + lane_base, a);
                        tmem_ld16(tB + half * 32 + q0 + lane_base, b);
                        tmem_wait_ld();
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float2 r =
                                fma_f32x2(make_float2(ej, ej),
                                          make_float2(__uint_as_float(a[2 * q]), __uint_as_float(a[2 * q + 1])),
                                          make_float2(__uint_as_float(b[2 * q]), __uint_as_float(b[2 * q + 1])));
                            const uint4 &v = zv[q0 / 8 + q / 4];
                            const uint32_t zz = (q & 3) == 0 ? v.x : (q & 3) == 1 ? v.y : (q & 3) == 2 ? v.z : v.w;
                            const float z0 = bf16lo(zz), z1 = bf16hi(zz);
                            g[q0 + 2 * q] = r.x * silu_approx(z0);
                            g[q0 + 2 * q + 1] = r.y * silu_approx(z1);
                        }
                    }
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pb.acc_free);
                    float sa[4] = {0.f, 0.f, 0.f, 0.f};  // four partial sums: shorter dependent chains
#pragma unroll
                    for (int q = 0; q < 32; ++q) sa[q & 3] += g[q];
                    const float m = ((sa[0] + sa[1]) + (sa[2] + sa[3])) * (1.f / 32);
#pragma unroll
                    for (int k = 0; k < 4; ++k) sa[k] = 0.f;
#pragma unroll
                    for (int q = 0; q < 32; ++q) sa[q & 3] = fmaf(g[q] - m, g[q] - m, sa[q & 3]);
                    const float m2 = (sa[0] + sa[1]) + (sa[2] + sa[3]);
                    float2 *sStat = reinterpret_cast<float2 *>(smem + kOffStat) + pl * 2 * kRows;
                    sStat[half * kRows + lrow] = make_float2(m, m2);
                    if (wtid < 32) cp_async_wait_all();  // the weight and bias, published by the barrier
                    named_bar_sync(bar_id, kPipeThreads);
                    const float2 o = sStat[(1 - half) * kRows + lrow];
                    const float dm = m - o.x;
                    const float mean = 0.5f * (m + o.x);
                    const float rstd = rsqrtf(fmaf(16.f * dm, dm, m2 + o.y) * (1.f / 64) + p.eps);
                    const float4 *wp = p.gw ? reinterpret_cast<const float4 *>(sWB + half * 32) : nullptr;
                    const float4 *bp = p.gb ? reinterpret_cast<const float4 *>(sWB + kP + half * 32) : nullptr;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint32_t o4[4];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int q = 8 * k + 4 * e;
                            const float4 wv = wp ? wp[q / 4] : make_float4(1.f, 1.f, 1.f, 1.f);
                            const float4 bv = bp ? bp[q / 4] : make_float4(0.f, 0.f, 0.f, 0.f);
                            o4[2 * e] = pack_bf16x2(fmaf((g[q] - mean) * rstd, wv.x, bv.x),
                                                    fmaf((g[q + 1] - mean) * rstd, wv.y, bv.y));
                            o4[2 * e + 1] = pack_bf16x2(fmaf((g[q + 2] - mean) * rstd, wv.z, bv.z),
                                                        fmaf((g[q + 3] - mean) * rstd, wv.w, bv.w));
                        }
                        sts128(sW + swz(lrow, half * 4 + k), make_uint4(o4[0], o4[1], o4[2], o4[3]));
                    }
                    fence_view_async_shared();
                    named_bar_sync(bar_id, kPipeThreads);
                    if (ctl) {
                        tma_store_4d(&mY, sW, 0, h, un.t0 + un.row0, un.b);
                        bulk_commit();
                        if (has_next && (own || kD > 1) && un.c > 0)
                            ready_seen = ld_acquire_gpu(inc_flag<kD>(p.inc, bh + 2, un.c - 1));
                    }
                } else {
#pragma unroll
                    for (int q0 = 0; q0 < 32; q0 += 16) {
                        uint32_t a[16], b[16];
                        tmem_ld16(tA + half * 32 + q0 + lane_base, a);
                        tmem_ld16(tB + half * 32 + q0 + lane_base, b);
                        tmem_wait_ld();
                        uint32_t o[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            float2 r =
                                fma_f32x2(make_float2(ej, ej),
                                          make_float2(__uint_as_float(a[2 * q]), __uint_as_float(a[2 * q + 1])),
                                          make_float2(__uint_as_float(b[2 * q]), __uint_as_float(b[2 * q + 1])));
                            if (kAccum) {
                                const uint4 &v = yprev[q0 / 8 + q / 4];
                                const uint32_t w = (q & 3) == 0 ? v.x : (q & 3) == 1 ? v.y : (q & 3) == 2 ? v.z : v.w;
                                r.x += bf16lo(w);
                                r.y += bf16hi(w);
                            }
                            o[q] = pack_bf16x2(r.x, r.y);
                        }
                        const int ch = half * 4 + q0 / 8;
                        sts128(sW + swz(lrow, ch), make_uint4(o[0], o[1], o[2], o[3]));
                        sts128(sW + swz(lrow, ch + 1), make_uint4(o[4], o[5], o[6], o[7]));
                    }
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pb.acc_free);
                    fence_view_async_shared();
                    named_bar_sync(bar_id, kPipeThreads);
                    if (ctl) {
                        tma_store_4d(&mY, sW, 0, h, un.t0 + un.row0, un.b);
                        bulk_commit();
                        if (has_next && (own || kD > 1) && un.c > 0)
                            ready_seen = ld_acquire_gpu(inc_flag<kD>(p.inc, bh + 2, un.c - 1));
                    }
                }
            }
        }
        if (ctl) bulk_wait_all();
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
bool fused_supported(const Shape &sh, int dtype) {
    return dtype == SSD_BF16 && sh.P % 8 == 0 && (sh.P <= kP || sh.P == 2 * kP) &&
           ((sh.N >= 16 && sh.N <= 128 && sh.N % 16 == 0) || sh.N == 256) &&
           (sh.Q == 128 || sh.Q == 256);
}

static int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

// Heads per work unit: enough to amortise the unit's C, B and G over several heads (they are loaded
// and formed once per unit), few enough that every SM gets several units.  Up to 8 for the other
// blocks and 4 for the owners' block, whose heads take about twice as long; with look-back (long
// sequences, few heads) owners' units of 2 heads, one per pipeline: a unit's later heads would otherwise
// wait behind its first head's chain step, and the chunks in flight would advance at that pace.  The
// other blocks read a state their chunk's predecessor published well before, so theirs stay large.
static int heads_per_unit(const Shape &sh, bool lookback, bool owners) {
    const int hpg = sh.heads_per_group, most = owners ? (lookback ? 2 : 4) : 8;
    if (hpg <= most) return hpg;
    const int blocks = (hpg + most - 1) / most;
    return (hpg + blocks - 1) / blocks;
}

// One launch of the fused kernel, worked out on the host ahead of the call's first enqueued operation
// (so that the GPU does not wait on tensor-map encoding between the workspace clear and the launch).
// Held per host thread: a call prepares its launches and enqueues them before it returns.
namespace {
using FusedKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, Params);
struct FusedLaunch {
    CUtensorMap mC, mB, mX, mY, mR;
    Params p;
    FusedKernel kernel;
    int grid;
};
thread_local FusedLaunch g_launch[kMaxFusedPasses];
}  // namespace

// Prepares launch `slot` of the fused kernel for state columns [n_half * 128, ...) and head columns
// [p_half * 64, ...) of the problem `full` (all of them when full.N <= 128 and full.P <= 64).  The second
// half of a 256-wide state adds to the y of the first.
// `pw` is this launch's part of the workspace, laid out as `w`; the status word is shared.
cudaError_t prepare_ssd_fused(const __nv_bfloat16 *x, const float *dt, const float *A, const __nv_bfloat16 *B,
                              const __nv_bfloat16 *C, const float *D, const float *init, float *fin, char *pw,
                              const Workspace &w, int *status, __nv_bfloat16 *y, const Shape &full, int p_half,
                              int n_half, const FusedDebug *dbg, const FusedGate *gate, int slot) {
    if (slot < 0 || slot >= kMaxFusedPasses) return cudaErrorInvalidValue;
    FusedLaunch &L = g_launch[slot];
    // the gate needs the whole row of a head in one launch
    if (gate && (full.P != kP || full.N > 128)) return cudaErrorInvalidValue;
    Shape sh = full;
    const int n_off = n_half * 128, p_off = p_half * kP;
    if (full.N > 128) sh.N = 128;
    sh.P = kP;
    CUtensorMap &mC = L.mC, &mB = L.mB, &mX = L.mX, &mY = L.mY, &mR = L.mR;
    const uint64_t dbc[4] = {(uint64_t)sh.N, (uint64_t)sh.G, (uint64_t)sh.T, (uint64_t)sh.batch};
    const uint64_t sbc[3] = {(uint64_t)full.N * 2, (uint64_t)sh.G * full.N * 2,
                             (uint64_t)sh.T * sh.G * full.N * 2};
    B += n_off;
    C += n_off;
    const uint32_t box[4] = {64, 1, kRows, 1};
    // x and y: the launch's 64 head columns (fewer when P < 64: loads past P read zero, stores are clipped)
    const uint64_t dx[4] = {(uint64_t)min(kP, full.P - p_off), (uint64_t)sh.H, (uint64_t)sh.T, (uint64_t)sh.batch};
    const uint64_t sx[3] = {(uint64_t)full.P * 2, (uint64_t)sh.H * full.P * 2, (uint64_t)sh.T * sh.H * full.P * 2};
    x += p_off;
    y += p_off;
    if (!make_map_bf16(&mC, C, 4, dbc, sbc, box) || !make_map_bf16(&mB, B, 4, dbc, sbc, box) ||
        !make_map_bf16(&mX, x, 4, dx, sx, box) || !make_map_bf16(&mY, y, 4, dx, sx, box))
        return cudaErrorInvalidValue;
    Params &p = L.p;
    p = Params{};
    p.sh = sh;
    p.dt = dt;
    p.A = A;
    p.D = (n_half == 0) ? D : nullptr;
    p.state_ld = full.N;
    p.n_off = n_off;
    p.z = gate ? static_cast<const __nv_bfloat16 *>(gate->z) : nullptr;
    p.gw = gate ? gate->weight : nullptr;
    p.gb = gate ? gate->bias : nullptr;
    p.eps = gate ? gate->eps : 0.f;
    p.p_full = full.P;
    p.p_off = p_off;
    p.init = init;
    p.fin = fin;
    p.ring = reinterpret_cast<float *>(pw + w.ring_off);
    p.tile_rows = fused_tile_rows(sh);
    p.inc = reinterpret_cast<int *>(pw + w.inc_off);
    p.tin = reinterpret_cast<int *>(pw + w.tin_off);
    p.agg = reinterpret_cast<int *>(pw + w.agg_off);
    p.cons = reinterpret_cast<int *>(pw + w.cons_off);
    p.sig = reinterpret_cast<float *>(pw + w.sig_off);
    p.counter = reinterpret_cast<int *>(pw + w.counter_off);
    p.status = status;
    p.y = y;
    p.NK = (sh.N + 63) / 64;
    p.halves = sh.Q / kRows;

    const bool lookback = fused_lookback(sh) == 4;  // the workspace's layout has the same shape
    // the bf16 state tiles without look-back: [b*H*3][tile_rows][64], one TMA box per tile (with
    // look-back there are none and the map, over the fp32 ring, is never used)
    {
        const uint64_t slots = lookback ? 1 : (uint64_t)sh.batch * sh.H * fused_ring_slots(1);
        const uint64_t dr[3] = {(uint64_t)kP, (uint64_t)p.tile_rows, slots};
        const uint64_t sr[2] = {(uint64_t)kP * 2, (uint64_t)p.tile_rows * kP * 2};
        const uint32_t boxr[3] = {(uint32_t)kP, (uint32_t)p.tile_rows, 1};
        if (!make_map_bf16(&mR, pw + (lookback ? w.ring_off : w.tile_off), 3, dr, sr, boxr))
            return cudaErrorInvalidValue;
    }
    for (int r = 0; r < 2; ++r) {
        p.hpu[r] = heads_per_unit(sh, lookback, r == 1 && p.halves == 2);
        p.blocks[r] = (sh.heads_per_group + p.hpu[r] - 1) / p.hpu[r];
        p.units[r] = sh.batch * sh.G * p.blocks[r];
    }
    p.n_units = sh.nc * (p.halves == 2 ? p.units[0] + p.units[1] : p.units[0]);
    p.flag_polls = (dbg && dbg->flag_polls) ? dbg->flag_polls : kDefaultFlagPolls;
    p.withhold_bh = dbg ? dbg->withhold_bh : -1;
    p.withhold_c = dbg ? dbg->withhold_c : -1;
    auto kernel = gate ? (lookback ? ssd_fused_kernel<false, 4, true> : ssd_fused_kernel<false, 1, true>)
                  : (n_half > 0) ? (lookback ? ssd_fused_kernel<true, 4, false> : ssd_fused_kernel<true, 1, false>)
                                 : (lookback ? ssd_fused_kernel<false, 4, false> : ssd_fused_kernel<false, 1, false>);
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    L.kernel = kernel;
    L.grid = min(p.n_units, device_sm_count());
    return cudaSuccess;
}

// The clear of each launch's counter, flags and status before a call (`passes` regions `stride` bytes
// apart, `bytes` each, 16-byte multiples): it lets its dependent launch start at once, so that the fused
// kernel's start-up overlaps it (the fused kernel waits for it to complete before any global access).
__global__ void __launch_bounds__(256) fused_clear_kernel(char *ws, size_t stride, size_t bytes) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    uint4 *q = reinterpret_cast<uint4 *>(ws + blockIdx.y * stride);
    const size_t n = bytes / 16;
    for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (size_t)gridDim.x * 256)
        q[i] = make_uint4(0u, 0u, 0u, 0u);
}

cudaError_t enqueue_fused_clear(char *ws, size_t stride, size_t bytes, int passes, cudaStream_t st) {
    if (bytes % 16 != 0 || passes < 1 || passes > kMaxFusedPasses) return cudaErrorInvalidValue;
    const size_t blocks = std::min<size_t>(std::max<size_t>((bytes / 16 + 1023) / 1024, 1), 64);
    fused_clear_kernel<<<dim3((unsigned)blocks, (unsigned)passes), 256, 0, st>>>(ws, stride, bytes);
    return cudaGetLastError();
}

// Enqueues launch `slot` as prepared by this host thread's last prepare_ssd_fused for it; `after_clear`:
// it directly follows enqueue_fused_clear in the stream and may start while the clear runs.
cudaError_t enqueue_ssd_fused(int slot, bool after_clear, cudaStream_t st) {
    if (slot < 0 || slot >= kMaxFusedPasses) return cudaErrorInvalidValue;
    const FusedLaunch &L = g_launch[slot];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)L.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_clear ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, L.kernel, L.mC, L.mB, L.mX, L.mY, L.mR, L.p);
}

}  // namespace ssd
