// ssd_bwd_tc.cu -- the backward's masked chunk scans on the tensor cores (tcgen05, TMEM, TMA).
//
// The same operation as masked_scan_kernel in ssd_bwd.cu, per (chunk, 128-row block, head) tile:
//
//   out_r[w] = e_r * sum_k R_r[k] St[k][w]
//            + sum_{i in chunk, i >= r (kAnti) or i <= r} exp(+-(s_i - s_r)) (R_r . K_i) V_i[w]
//            + D_h V_r[w]                                          (when D is given)
//
// with e_r = exp(s_end - s_r) (kAnti) or exp(s_r).  It is the adjoint of the forward's block decomposition
// ("Transformers are SSMs", analysis page, section "The Block-Decomposition SSD Algorithm"): the quadratic
// (masked) form inside a chunk and the state term across chunks, here with given chunk states instead of
// a chain.  The products run as bf16 x bf16 -> fp32 MMAs, over the chunk's columns on the mask's side of
// the block (128 or 256 of them) in halves of 128:
//
//   G    = R_blk K_half^T        (M = 128 rows, N = 128, K = KD)
//   M    = G o exp(+-(s_i - s_r)) on the triangle, bf16, in tensor memory (built by the CUDA-core warps)
//   acc += M V_half              (A from tensor memory, N = W)
//   acc2 = R_blk St^T            (the state tile [k][w] in bf16, built by the CUDA-core warps; N = W)
//   out  = e_r acc2 + acc (+ D V_r), one row per thread, stored from registers.
//
// For the per-head dB and dC terms the mask and the state tile also enter as bf16 low parts (what the
// rounding to bf16 left out), so those products are as accurate as fp32 accumulation allows.  Those terms
// are summed over each group's heads in registers (dB = sum_h dB^(h), dC likewise) rather than stored:
// each CTA takes a contiguous, cost-balanced run of tiles, head innermost, stores one partial sum per
// (chunk, block, group) it touched plus each head's rows dotted with B or C (which dsigma needs), and
// head_sum_reduce_kernel adds the partial sums of the few CTAs that share a (chunk, block, group).
// Shapes: KD, W in {64, 128}; Q in {128, 256}; R, K, V bf16 rows of [batch][T][heads or groups][dim].
// Tensor memory (512 columns): G at 0, the mask at 128 (its low part at 192), acc at 256, acc2 at 384.
// One persistent CTA per SM (it takes all of tensor memory) taking every grid-th tile; while its warps
// drain one tile, the next tile's loads and G product run.  9 warps: 0-7 CUDA-core work (two warpgroups
// over the 128 lanes, each half of the columns), 8 TMA and MMA issue.  Every wait is bounded (about 2 s of
// %globaltimer, 1 ms once any CTA has given up): on expiry the CTA records SSD_ERR_TIMEOUT in the status
// word, and the issuer still waits (bounded) for its own MMAs before tensor memory is freed.
#include <algorithm>

#include "ssd_common.cuh"
#include "tc_prims.cuh"
#include "tma_host.h"

namespace ssd {

using namespace tc;

namespace bt {

constexpr int kRows = 128;
constexpr int kCudaWarps = 8;
constexpr int kThreads = 32 * kCudaWarps + 32;
constexpr uint32_t kTmemCols = 512;
// tensor memory: G of one 128-column half at 0; the half's mask at 128 (bf16; its low part at 192 when
// split); acc at 256; acc2 at 384
constexpr uint32_t kColG = 0, kColMhi = 128, kColMlo = 192, kColAcc = 256, kColAcc2 = 384;
// shared memory (1 KiB aligned): R [KD/64 atoms][128 rows], K and V [atoms][256 rows], the state tile
// [W/64 atoms][KD rows] and its low part, prefix sums [256]
constexpr uint32_t kOffR = 0;           // 2 x 16 KiB
constexpr uint32_t kOffK = 32768;       // 2 x 32 KiB
constexpr uint32_t kOffV = 98304;       // 2 x 32 KiB
constexpr uint32_t kOffSt = 163840;     // 2 x 16 KiB
constexpr uint32_t kOffStLo = 196608;   // 2 x 8 KiB (split: KD = 64)
constexpr uint32_t kOffS = 212992;      // two buffers of 256 floats (this tile's and the next one's)
constexpr uint32_t kOffF = kOffS + 2048;  // 256 floats: the mask's column factors
constexpr uint32_t kSmemBytes = kOffF + 1024 + 1024;
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;

// Contiguous, cost-balanced ranges of (chunk, 128-row block, head) tiles, head innermost, for the scans
// that sum their per-head terms over each group's heads: CTA i takes the tiles whose cost before them lies
// in [i, i + 1) * total / ncta.  A tile costs its number of 128-column halves plus one (the state product
// and the drain), nothing for a block past a ragged chunk's end.  The host works the ranges out
// (TilePart) and hands the kernels their starts (TileRanges): a CTA reads its run from the table, and
// the sum over the CTAs' partial results finds which CTAs took part of a (chunk, block, group) by
// intersecting the runs with the group's tiles.
struct TileRanges {
    int ncta;
    int beg[kBwdSumMaxCtas + 1];  // first tile of CTA i; beg[ncta] = the tile count
};

struct TilePart {
    int H, Q, nc, blocks, len_last, ncta, anti;
    long long cfull, perseq, tiles, ctot;
    int cost_len(int len, int rb) const {
        const int r0 = rb * kRows;
        return r0 >= len ? 0 : 1 + (anti ? Q - r0 : r0 + kRows) / kRows;
    }
    int cost(int c, int rb) const { return cost_len(c == nc - 1 ? len_last : Q, rb); }
    void init(const Shape &sh, bool is_anti, int n) {
        H = sh.H;
        Q = sh.Q;
        nc = sh.nc;
        blocks = sh.Q / kRows;
        len_last = sh.T - (sh.nc - 1) * sh.Q;
        ncta = n;
        anti = is_anti ? 1 : 0;
        cfull = 0;
        long long clast = 0;
        for (int rb = 0; rb < blocks; ++rb) {
            cfull += cost_len(Q, rb);
            clast += cost_len(len_last, rb);
        }
        perseq = (long long)(nc - 1) * cfull + clast;
        tiles = (long long)sh.batch * nc * blocks * H;
        ctot = (long long)sh.batch * perseq * H;
    }
    // cost of the tiles before tile t (t = tiles gives the total)
    long long cum(long long t) const {
        const long long blk = t / H;
        const int h = (int)(t - blk * H), rb = (int)(blk % blocks);
        const long long r = blk / blocks;
        const int c = (int)(r % nc);
        const long long b = r / nc;
        long long before = b * perseq + (long long)c * cfull;
        for (int q = 0; q < rb; ++q) before += cost(c, q);
        return before * H + (long long)cost(c, rb) * h;
    }
    // first tile of CTA i (i = ncta gives the end): the first tile whose cost before it reaches i / ncta
    // of the total
    long long beg(int i) const {
        if (i <= 0) return 0;
        if (i >= ncta) return tiles;
        long long lo = 0, hi = tiles;
        const long long want = (long long)i * ctot;
        while (lo < hi) {
            const long long mid = (lo + hi) / 2;
            if (cum(mid) * ncta >= want) hi = mid;
            else lo = mid + 1;
        }
        return lo;
    }
    void ranges(TileRanges *r) const {
        r->ncta = ncta;
        for (int i = 0; i <= ncta; ++i) r->beg[i] = (int)beg(i);
    }
};

struct Args {
    const float *s;    // [batch][H][nc][Q] chunk prefix sums of dt * A (natural units)
    const float *St;   // [batch][nc][H][P * N]: read as [KD][W] (st_kw) or [W][KD]
    int st_kw;
    const float *D;    // per head, or null
    const __nv_bfloat16 *V;  // for the D term (row r of V), [batch][T][heads or groups][W]
    int v_head;
    void *out;         // [batch][T][H][W], bf16 (kOutBf16) or fp32
    int *status;
    Shape sh;
    // head sums (kSum): the row each term is dotted with ([batch][T][G][W], bf16), the two column halves'
    // dot products [batch][H][T][2], the CTAs' partial sums [CTA + (chunk, block, group) key][128][W], and
    // the tile ranges
    const __nv_bfloat16 *dotv;
    float *dotp;
    float *part;
    TileRanges tr;
};

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait on one of the CTA's own barriers (its producers are its own TMA, MMAs and warps, so only a
// defect of the kernel can make it expire).  Once any CTA has given up (the status word is set) the limit
// drops to 1 ms, so that a defect common to every CTA still ends the grid in seconds.
constexpr uint64_t kBrokenWaitNs = 1000000ull;
__device__ __forceinline__ void wait_bar(uint64_t *bar, uint32_t parity, int *status) {
    if (mbar_try_wait(bar, parity)) return;
    const uint64_t t0 = global_ns(), limit = ld_relaxed_gpu(status) ? kBrokenWaitNs : kWaitNs;
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > limit) {
            atomicExch(status, SSD_ERR_TIMEOUT);
            return;
        }
    }
}

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    return (uint32_t)row * 128u + ((uint32_t)(chunk ^ (row & 7)) << 4);
}

// bf16 pair of (a, b) and, for the split operands, the pair of what rounding left out
__device__ __forceinline__ uint32_t pack_lo(float a, float b, uint32_t hi) {
    return pack_bf16x2(a - bf16lo(hi), b - bf16hi(hi));
}

}  // namespace bt

using namespace bt;

// kSplit: the mask and the state tile enter the products as a bf16 high part plus a bf16 low part (two
// MMAs each); R, K and V are bf16 inputs and exact, so the products are then as accurate as fp32
// accumulation allows.  Used for the per-head dB and dC terms, from which the dt, A and D gradients follow
// through differences of large terms.
// kSum: the per-head terms are not stored; each CTA takes a contiguous run of tiles (TilePart), adds each
// head's rows into registers in head order and stores the sum once per (chunk, block, group) it touched,
// plus each head's row dotted with the row of a.dotv (the two column halves apart).
template <int KD, int W, bool kAnti, bool kOutBf16, bool kSplit, bool kSum>
__global__ void __launch_bounds__(bt::kThreads, 1)
    masked_scan_tc_kernel(const __grid_constant__ CUtensorMap mR, const __grid_constant__ CUtensorMap mK,
                          const __grid_constant__ CUtensorMap mV, const __grid_constant__ bt::Args a, int r_head,
                          int k_head,
                          int v_head) {
    static_assert(!kSplit || KD == 64, "the low part of the state tile has room for KD = 64");
    static_assert(KD == 64 || W == 64, "the fp32 state is staged in the unused second atom of K or V");
    static_assert(!kSum || !kOutBf16, "head sums are fp32");
    // the fp32 state [KD][W] (32 KB), copied in asynchronously: the K region's second atom (KD = 64) or the
    // V region's (W = 64), which this shape leaves unused
    constexpr uint32_t kOffRaw = (KD == 64) ? kOffK + 32768 : kOffV + 32768;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t ld_full, ld_v, g_done, st_full, m_full, mx_done, fin_done, acc_free;
    __shared__ uint32_t tslot;
    const Shape &sh = a.sh;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int blocks = sh.Q / kRows;
    // this CTA's tiles (chunk, 128-row block, head): every gridDim.x-th, so that each CTA gets the same mix
    // of one- and two-half blocks; for head sums a contiguous run of about equal cost
    const int tiles = sh.batch * sh.nc * blocks * sh.H;
    const int t_beg = kSum ? a.tr.beg[blockIdx.x] : (int)blockIdx.x;
    const int t_end = kSum ? a.tr.beg[blockIdx.x + 1] : tiles;
    const int t_step = kSum ? 1 : (int)gridDim.x;
    if (t_beg >= t_end) return;  // whole CTA
    auto tile = [&](int t, int &b, int &c, int &rb, int &h) {
        h = t % sh.H;
        int r = t / sh.H;
        rb = r % blocks;
        r /= blocks;
        c = r % sh.nc;
        b = r / sh.nc;
    };

    if (warp == 0) tmem_alloc(&tslot, kTmemCols);
    if (tid == 0) {
        mbar_init(&ld_full, 1);
        mbar_init(&ld_v, 1);
        mbar_init(&g_done, 1);
        mbar_init(&mx_done, 1);
        mbar_init(&fin_done, 1);
        mbar_init(&st_full, kCudaWarps);
        mbar_init(&m_full, kCudaWarps);
        mbar_init(&acc_free, kCudaWarps);
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    uint8_t *sR = smem + kOffR, *sK = smem + kOffK, *sV = smem + kOffV, *sSt = smem + kOffSt;
    uint8_t *sStLo = smem + kOffStLo;
    float *sq = reinterpret_cast<float *>(smem + kOffS);

    if (warp == kCudaWarps) {
        // ---------------- TMA and MMA issue (lane 0) ----------------
        // Every barrier phase is counted on both sides; one tile's last MMA (fin_done) completes before the
        // next tile's loads, and its G and masked products may run while the warps drain the tile before.
        if (lane == 0) {
            uint32_t n_ld = 0, n_v = 0, n_m = 0, n_st = 0, n_fin = 0, n_free = 0;
            long long rk_key = -1, v_key = -1;  // the group-shared operands now in shared memory
            const uint32_t idG = idesc_bf16_f32(kRows, kRows, 0, 0);  // R (K-major) x K rows (K-major)
            const uint32_t idW = idesc_bf16_f32(kRows, W, 0, 1);      // x V [i][w] or the state tile [k][w]
            for (int t = t_beg; t < t_end; t += t_step) {
                int b, c, rb, h;
                tile(t, b, c, rb, h);
                const int g = h / sh.heads_per_group;
                const int t0 = c * sh.Q, len = min(sh.Q, sh.T - t0), r0 = rb * kRows;
                if (r0 >= len) continue;  // a block past a ragged chunk's end
                const int cbeg = kAnti ? r0 : 0;
                const int nh = (kAnti ? sh.Q - r0 : r0 + kRows) / kRows;  // 1 or 2
                const int hr = r_head ? h : g, hk = k_head ? h : g, hv = v_head ? h : g;
                const long long gkey = (((long long)b * sh.nc + c) * blocks + rb) * sh.G + g;
                // R and K (for G), kept while they are the group's and the block is the same
                const bool new_rk = r_head || k_head || gkey != rk_key;
                if (new_rk) {
                    mbar_arrive_expect_tx(&ld_full, (uint32_t)(KD / 64) * (1u + (uint32_t)nh) * 16384u);
                    for (int k = 0; k < KD / 64; ++k) {
                        tma_load_4d(sR + k * 16384, &mR, &ld_full, k * 64, hr, t0 + r0, b);
                        for (int q = 0; q < nh; ++q)
                            tma_load_4d(sK + k * 32768 + q * 16384, &mK, &ld_full, k * 64, hk, t0 + cbeg + q * kRows,
                                        b);
                    }
                    rk_key = (r_head || k_head) ? -1 : gkey;
                }
                const bool new_v = v_head || gkey != v_key;
                if (new_v) {
                    mbar_arrive_expect_tx(&ld_v, (uint32_t)(W / 64) * (uint32_t)nh * 16384u);
                    for (int k = 0; k < W / 64; ++k)
                        for (int q = 0; q < nh; ++q)
                            tma_load_4d(sV + k * 32768 + q * 16384, &mV, &ld_v, k * 64, hv, t0 + cbeg + q * kRows, b);
                    v_key = v_head ? -1 : gkey;
                }
                if (new_rk) wait_bar(&ld_full, n_ld++ & 1, a.status);
                fence_after_sync();
                for (int ch = 0; ch < nh; ++ch) {
                    // G of this half into columns 0..127 (the warps have read the previous half's: m_full)
                    for (int kk = 0; kk < KD / 16; ++kk) {
                        const int atom = kk >> 2, kin = kk & 3;
                        mma_ss(tmem + kColG, smem_desc_sw128(smem_u32(sR) + atom * 16384 + kin * 32, 16, 1024),
                               smem_desc_sw128(smem_u32(sK) + atom * 32768 + ch * 16384 + kin * 32, 16, 1024), idG,
                               kk > 0);
                    }
                    mma_commit(&g_done);
                    if (ch == 0 && new_v) wait_bar(&ld_v, n_v++ & 1, a.status);
                    // acc += M V over the half's 128 rows of V (A from tensor memory), once the mask is in and
                    // (first half) the previous tile's drain has read both accumulators
                    wait_bar(&m_full, n_m++ & 1, a.status);
                    if (ch == 0 && n_fin > 0) wait_bar(&acc_free, n_free++ & 1, a.status);
                    fence_after_sync();
                    for (int kk = 0; kk < kRows / 16; ++kk) {
                        const uint64_t vd = smem_desc_sw128(smem_u32(sV) + ch * 16384 + kk * 2048, 32768, 1024);
                        mma_ts(tmem + kColAcc, tmem + kColMhi + kk * 8, vd, idW, ch > 0 || kk > 0);
                        if (kSplit) mma_ts(tmem + kColAcc, tmem + kColMlo + kk * 8, vd, idW, 1);
                    }
                    mma_commit(&mx_done);
                }
                // acc2 = R St^T
                wait_bar(&st_full, n_st++ & 1, a.status);
                fence_after_sync();
                for (int kk = 0; kk < KD / 16; ++kk) {
                    const int atom = kk >> 2, kin = kk & 3;
                    const uint64_t rd = smem_desc_sw128(smem_u32(sR) + atom * 16384 + kin * 32, 16, 1024);
                    mma_ss(tmem + kColAcc2, rd, smem_desc_sw128(smem_u32(sSt) + kk * 2048, 16384, 1024), idW, kk > 0);
                    if (kSplit)
                        mma_ss(tmem + kColAcc2, rd, smem_desc_sw128(smem_u32(sStLo) + kk * 2048, 8192, 1024), idW, 1);
                }
                mma_commit(&fin_done);
                // the tile's products are done before its R, K or V are replaced (and nothing is in flight
                // when the CTA leaves)
                wait_bar(&fin_done, n_fin++ & 1, a.status);
            }
        }
        __syncwarp();
    } else {
        // ---------------- CUDA-core warps ----------------
        const int wq = warp & 3, half = warp >> 2;  // TMEM lane quarter, column half
        const int lrow = wq * 32 + lane;            // this thread's row of the block
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        float *sRaw = reinterpret_cast<float *>(smem + kOffRaw);
        float *const sqb[2] = {sq, sq + 256};
        uint32_t n_g = 0, n_mx = 0, n_fin = 0;
        float hs[kSum ? W / 2 : 1];  // head sums: this thread's row, its half of the columns
        int seg = -1;                // the (chunk, block, group) key they belong to
        auto valid = [&](int t) {
            int b, c, rb, h;
            tile(t, b, c, rb, h);
            return rb * kRows < min(sh.Q, sh.T - c * sh.Q);
        };
        // the prefix sums of tile t into buffer d, one 4-byte async copy per token, as one commit group
        auto request_sq = [&](int t, float *d) {
            int b, c, rb, h;
            tile(t, b, c, rb, h);
            const float *sch = a.s + (((size_t)b * sh.H + h) * sh.nc + c) * sh.Q;
            for (int i = tid; i < sh.Q; i += 32 * kCudaWarps) cp_async4(d + i, sch + i);
            cp_async_commit();
        };
        int t = t_beg;
        while (t < t_end && !valid(t)) t += t_step;
        if (t < t_end) request_sq(t, sqb[0]);
        for (int k = 0; t < t_end; ++k) {
            int tn = t + t_step;
            while (tn < t_end && !valid(tn)) tn += t_step;
            int b, c, rb, h;
            tile(t, b, c, rb, h);
            const int g = h / sh.heads_per_group;
            const int t0 = c * sh.Q, len = min(sh.Q, sh.T - t0), r0 = rb * kRows;
            const int cbeg = kAnti ? r0 : 0;
            const int nh = (kAnti ? sh.Q - r0 : r0 + kRows) / kRows;
            const int j = r0 + lrow;  // row within the chunk
            const float *sq = sqb[k & 1];
            const int key = t / sh.heads_per_group;
            if (kSum && key != seg) {
#pragma unroll
                for (int e = 0; e < (kSum ? W / 2 : 1); ++e) hs[e] = 0.f;
                seg = key;
            }
            // every thread is done with the previous tile's staged state (and the prefix-sum buffer the next
            // tile's go to)
            named_bar_sync(1, 32 * kCudaWarps);
            // the fp32 state on its way into shared memory (async copies: no barrier waits for them, so
            // its DRAM latency passes while the masks are built), one commit group
            const float *Sp = a.St + (((size_t)b * sh.nc + c) * sh.H + h) * (size_t)sh.P * sh.N;
            for (int i = tid; i < KD * W / 4; i += 32 * kCudaWarps) cp_async16(sRaw + 4 * i, Sp + 4 * i);
            cp_async_commit();
            cp_async_wait_group<1>();           // this tile's prefix sums (requested during the tile before)
            named_bar_sync(1, 32 * kCudaWarps);  // everyone's are in
            const float sj = (j < len) ? sq[j] : 0.f;
            // the mask's column factors, relative to the column's 16-wide piece: exp(s_i - s_{piece start})
            // (anti-causal) or exp(s_{piece end} - s_i) (causal), both <= 1 for decaying inputs
            float *sFac = reinterpret_cast<float *>(smem + kOffF);
            if (tid < sh.Q)
                sFac[tid] = ex2((kAnti ? sq[tid] - sq[tid & ~15] : sq[tid | 15] - sq[tid]) * kLog2e);
            named_bar_sync(1, 32 * kCudaWarps);

            // the mask, one 128-column half at a time: this thread's row, its 64 of the half's columns
            const uint32_t mx0 = n_mx;
            for (int ch = 0; ch < nh; ++ch) {
                wait_bar(&g_done, n_g++ & 1, a.status);
                if (ch > 0) wait_bar(&mx_done, (mx0 + ch - 1) & 1, a.status);  // the previous half's mask was used
                fence_after_sync();
#pragma unroll 1
                for (int q0 = half * 64; q0 < half * 64 + 64; q0 += 16) {
                    uint32_t gv[16];
                    tmem_ld16(tmem + kColG + q0 + lane_base, gv);
                    tmem_wait_ld();
                    uint32_t o[8], ol[8];
                    // a piece of 16 columns wholly on the kept side of this row (and inside the chunk) takes a
                    // row factor times the column factors, one exponential per piece; a piece wholly on the
                    // other side is zero; a piece the diagonal or the chunk's end crosses takes one exponential
                    // per element
                    const int i0 = cbeg + ch * kRows + q0;  // the piece's first column within the chunk
                    const bool jv = j < len, whole = i0 + 15 < len;
                    const bool fac = jv && whole && (kAnti ? i0 >= j : i0 + 15 <= j);
                    const bool zero = !jv || (kAnti ? i0 + 15 < j : i0 > j);
                    if (fac) {
                        const float rf = ex2((kAnti ? sq[i0] - sj : sj - sq[i0 + 15]) * kLog2e);
                        const float4 *f4 = reinterpret_cast<const float4 *>(sFac + i0);
#pragma unroll
                        for (int e = 0; e < 16; e += 4) {
                            const float4 f = f4[e / 4];
                            const float m0 = __uint_as_float(gv[e]) * (rf * f.x);
                            const float m1 = __uint_as_float(gv[e + 1]) * (rf * f.y);
                            const float m2 = __uint_as_float(gv[e + 2]) * (rf * f.z);
                            const float m3 = __uint_as_float(gv[e + 3]) * (rf * f.w);
                            o[e / 2] = pack_bf16x2(m0, m1);
                            o[e / 2 + 1] = pack_bf16x2(m2, m3);
                            if (kSplit) {
                                ol[e / 2] = pack_lo(m0, m1, o[e / 2]);
                                ol[e / 2 + 1] = pack_lo(m2, m3, o[e / 2 + 1]);
                            }
                        }
                    } else if (zero) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) o[e] = ol[e] = 0u;
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; e += 2) {
                            float m[2];
#pragma unroll
                            for (int k = 0; k < 2; ++k) {
                                const int i = i0 + e + k;  // column within the chunk
                                const bool ok = i < len && (kAnti ? i >= j : i <= j);
                                m[k] = ok ? __uint_as_float(gv[e + k]) *
                                                ex2((kAnti ? sq[i] - sj : sj - sq[i]) * kLog2e)
                                          : 0.f;
                            }
                            o[e / 2] = pack_bf16x2(m[0], m[1]);
                            if (kSplit) ol[e / 2] = pack_lo(m[0], m[1], o[e / 2]);
                        }
                    }
                    tmem_st8(tmem + kColMhi + q0 / 2 + lane_base, o);
                    if (kSplit) tmem_st8(tmem + kColMlo + q0 / 2 + lane_base, ol);
                }
                tmem_wait_st();
                fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&m_full);
            }
            n_mx = mx0 + nh;
            // the next tile's prefix sums into the other buffer, while this tile's state tile and drain run
            if (tn < t_end) request_sq(tn, sqb[(k + 1) & 1]);

            // the state tile [k][w] in bf16 (and its low part), 128-byte swizzled, 64-wide w atoms of KD rows,
            // from the staged fp32 state (the previous tile's products, acc2 among them, are done: its drain
            // waited for them)
            if (tn < t_end)
                cp_async_wait_group<1>();  // the state (the newest group, the next prefix sums, may still fly)
            else
                cp_async_wait_group<0>();
            named_bar_sync(1, 32 * kCudaWarps);  // every thread's copies are in
            for (int idx = tid; idx < KD * (W / 8); idx += 32 * kCudaWarps) {
                const int k = idx / (W / 8), w0 = (idx - k * (W / 8)) * 8;
                float v[8];
                if (a.st_kw) {
                    const float4 u0 = *reinterpret_cast<const float4 *>(sRaw + k * W + w0);
                    const float4 u1 = *reinterpret_cast<const float4 *>(sRaw + k * W + w0 + 4);
                    v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w;
                    v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] = sRaw[(w0 + e) * KD + k];
                }
                const uint4 tt = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                            pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
                *reinterpret_cast<uint4 *>(sSt + (w0 >> 6) * 16384 + swz(k, (w0 & 63) >> 3)) = tt;
                if (kSplit) {
                    const uint4 tl = make_uint4(pack_lo(v[0], v[1], tt.x), pack_lo(v[2], v[3], tt.y),
                                                pack_lo(v[4], v[5], tt.z), pack_lo(v[6], v[7], tt.w));
                    *reinterpret_cast<uint4 *>(sStLo + (w0 >> 6) * 8192 + swz(k, (w0 & 63) >> 3)) = tl;
                }
            }
            fence_view_async_shared();
            __syncwarp();
            if (lane == 0) mbar_arrive(&st_full);

            // the drain: out = e_r acc2 + acc (+ D V_r), this thread's row, its half of the W columns; the D
            // term's row of V (dx only) is loaded before the wait for the products, which covers its latency
            const size_t tok = (size_t)b * sh.T + t0 + j;
            const __nv_bfloat16 *vrow =
                a.V + (tok * (a.v_head ? sh.H : sh.G) + (a.v_head ? h : g)) * (size_t)W;
            const float Dh = a.D ? a.D[h] : 0.f;
            uint4 vr[(kOutBf16 || kSum) ? W / 16 : 1];
            if (kOutBf16 && a.D && j < len) {
                const uint4 *vp = reinterpret_cast<const uint4 *>(vrow + half * (W / 2));
#pragma unroll
                for (int q = 0; q < (kOutBf16 ? W / 16 : 1); ++q) vr[q] = vp[q];
            }
            if (kSum && j < len) {  // the row the head's term is dotted with
                const uint4 *vp =
                    reinterpret_cast<const uint4 *>(a.dotv + (tok * sh.G + g) * (size_t)W + half * (W / 2));
#pragma unroll
                for (int q = 0; q < (kSum ? W / 16 : 1); ++q) vr[q] = vp[q];
            }
            wait_bar(&fin_done, n_fin++ & 1, a.status);
            fence_after_sync();
            const float e_r = ex2((kAnti ? sq[sh.Q - 1] - sj : sj) * kLog2e);
            if constexpr (kSum) {
                float dot = 0.f;
#pragma unroll
                for (int q = 0; q < W / 32; ++q) {
                    uint32_t u[16], u2[16];
                    tmem_ld16(tmem + kColAcc + half * (W / 2) + q * 16 + lane_base, u);
                    tmem_ld16(tmem + kColAcc2 + half * (W / 2) + q * 16 + lane_base, u2);
                    tmem_wait_ld();
                    if (j >= len) continue;
                    const uint32_t ww[8] = {vr[2 * q].x, vr[2 * q].y, vr[2 * q].z, vr[2 * q].w,
                                            vr[2 * q + 1].x, vr[2 * q + 1].y, vr[2 * q + 1].z, vr[2 * q + 1].w};
#pragma unroll
                    for (int e = 0; e < 16; e += 2) {
                        const float r0v = fmaf(e_r, __uint_as_float(u2[e]), __uint_as_float(u[e]));
                        const float r1v = fmaf(e_r, __uint_as_float(u2[e + 1]), __uint_as_float(u[e + 1]));
                        hs[q * 16 + e] += r0v;
                        hs[q * 16 + e + 1] += r1v;
                        dot = fmaf(r0v, bf16lo(ww[e / 2]), dot);
                        dot = fmaf(r1v, bf16hi(ww[e / 2]), dot);
                    }
                }
                if (j < len) a.dotp[(((size_t)b * sh.H + h) * sh.T + t0 + j) * 2 + half] = dot;
            } else {
            for (int w0 = half * (W / 2); w0 < half * (W / 2) + W / 2; w0 += 16) {
                uint32_t u[16], u2[16];
                tmem_ld16(tmem + kColAcc + w0 + lane_base, u);
                tmem_ld16(tmem + kColAcc2 + w0 + lane_base, u2);
                tmem_wait_ld();
                if (j >= len) continue;
                float r[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) r[e] = fmaf(e_r, __uint_as_float(u2[e]), __uint_as_float(u[e]));
                if (a.D) {
                    const uint4 *vp = reinterpret_cast<const uint4 *>(vrow + w0);
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const uint4 vv = kOutBf16 ? vr[(w0 - half * (W / 2)) / 8 + q] : vp[q];
                        const uint32_t ww[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            r[8 * q + 2 * e] = fmaf(Dh, bf16lo(ww[e]), r[8 * q + 2 * e]);
                            r[8 * q + 2 * e + 1] = fmaf(Dh, bf16hi(ww[e]), r[8 * q + 2 * e + 1]);
                        }
                    }
                }
                if (kOutBf16) {
                    uint4 *op =
                        reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) + (tok * sh.H + h) * W + w0);
                    op[0] = make_uint4(pack_bf16x2(r[0], r[1]), pack_bf16x2(r[2], r[3]), pack_bf16x2(r[4], r[5]),
                                       pack_bf16x2(r[6], r[7]));
                    op[1] = make_uint4(pack_bf16x2(r[8], r[9]), pack_bf16x2(r[10], r[11]), pack_bf16x2(r[12], r[13]),
                                       pack_bf16x2(r[14], r[15]));
                } else {
                    float4 *op = reinterpret_cast<float4 *>(static_cast<float *>(a.out) + (tok * sh.H + h) * W + w0);
#pragma unroll
                    for (int q = 0; q < 4; ++q) op[q] = make_float4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
                }
            }
            }
            // both accumulators are read: the next tile's masked product may overwrite them
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_free);
            // the sums over the key's heads, once its last head in this CTA's run is in: slot CTA + key
            if (kSum && (tn >= t_end || tn / sh.heads_per_group != key) && j < len) {
                float4 *pp = reinterpret_cast<float4 *>(a.part + ((size_t)(blockIdx.x + key) * kRows + lrow) * W +
                                                        half * (W / 2));
#pragma unroll
                for (int q = 0; q < (kSum ? W / 8 : 0); ++q)
                    pp[q] = make_float4(hs[4 * q], hs[4 * q + 1], hs[4 * q + 2], hs[4 * q + 3]);
            }
            t = tn;
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Chunk states on the tensor cores: for every (chunk, head),
//
//   S[p][n] = sum_{i in chunk} w_i x_i[p] B_i[n],   w_i = exp(s_end - s_i), or exp(s_i) (from_start)
//
// the forward's stage 2 ("Transformers are SSMs", analysis page, section "The Block-Decomposition SSD
// Algorithm"), which the backward needs for the states entering every chunk, and (from the chunk's start,
// with dy and C) for the gradients arriving at them.  S^T = B^T (w o x) runs as one MMA chain (M = 128
// state columns n, N = 64 head columns p, K = the chunk's tokens, both operands MN-major); the weighted
// rows w_i x_i enter as a bf16 high part plus a bf16 low part, so the states carry fp32 accuracy into the
// gradients of dt, A and D.  Shapes: P = 64, N = 128, Q in {128, 256}; x [batch][T][H][64] and
// B [batch][T][G][128] bf16; S [batch][nc][H][64][128] fp32.
// ---------------------------------------------------------------------------
namespace cs {
constexpr uint32_t kOffB = 0;         // [2 n atoms][256 tokens] (32 KiB apart)
constexpr uint32_t kOffX = 65536;     // two buffers of [256 tokens][64 p] (32 KiB apart): the weighted rows' high part
constexpr uint32_t kOffXlo = 131072;  // two buffers of their low part
constexpr uint32_t kSmemBytes = 196608 + 1024;
}  // namespace cs

// Persistent: each CTA takes a contiguous run of `per_cta` (chunk, head) tiles, head fastest, so that B
// (shared by a group's heads) is loaded once per (batch, chunk, group) it meets.  x and its low part are
// double-buffered in shared memory and the accumulator in tensor memory (two 64-column halves), so that
// the CUDA-core warps drain tile k-1 while the tensor cores run tile k and the next x is on its way.
__global__ void __launch_bounds__(bt::kThreads, 1)
    chunk_state_tc_kernel(const __grid_constant__ CUtensorMap mX, const __grid_constant__ CUtensorMap mB,
                          const float *__restrict__ s, float *__restrict__ S, int *status, Shape sh,
                          int from_start, int per_cta) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t x_full[2], x_ready[2], done[2], acc_free[2], b_full;
    __shared__ uint32_t tslot;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tiles = sh.nc * sh.H * sh.batch;
    const int t_beg = blockIdx.x * per_cta, t_end = min(tiles, t_beg + per_cta);
    if (t_beg >= t_end) return;  // whole CTA
    const int nq = sh.Q / kRows;
    // tile t: head fastest, then chunk, then batch row
    auto tile = [&](int t, int &b, int &c, int &h) {
        h = t % sh.H;
        c = (t / sh.H) % sh.nc;
        b = t / (sh.H * sh.nc);
    };
    if (warp == 0) tmem_alloc(&tslot, 128);
    if (tid == 0) {
        for (int q = 0; q < 2; ++q) {
            mbar_init(&x_full[q], 1);
            mbar_init(&done[q], 1);
            mbar_init(&x_ready[q], kCudaWarps);
            mbar_init(&acc_free[q], kCudaWarps);
        }
        mbar_init(&b_full, 1);
        mbar_fence_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;
    uint8_t *sB = smem + cs::kOffB;
    if (warp == kCudaWarps) {
        if (lane == 0) {
            int cur_b = -1, cur_c = -1, cur_g = -1;
            uint32_t bcnt = 0;
            const uint32_t id = idesc_bf16_f32(kRows, 64, 1, 1);  // B^T (MN-major) x weighted rows (MN-major)
            for (int t = t_beg, k = 0; t < t_end; ++t, ++k) {
                int b, c, h;
                tile(t, b, c, h);
                const int g = h / sh.heads_per_group, buf = k & 1, t0 = c * sh.Q;
                uint8_t *sX = smem + cs::kOffX + buf * 32768, *sXlo = smem + cs::kOffXlo + buf * 32768;
                // this x buffer was last read by the product of tile k-2
                if (k >= 2) wait_bar(&done[buf], ((k - 2) >> 1) & 1, status);
                mbar_arrive_expect_tx(&x_full[buf], (uint32_t)nq * 16384u);
                for (int q = 0; q < nq; ++q) tma_load_4d(sX + q * 16384, &mX, &x_full[buf], 0, h, t0 + q * kRows, b);
                if (b != cur_b || c != cur_c || g != cur_g) {
                    // B was last read by the product of tile k-1
                    if (k >= 1) wait_bar(&done[(k - 1) & 1], ((k - 1) >> 1) & 1, status);
                    mbar_arrive_expect_tx(&b_full, (uint32_t)(2 * nq) * 16384u);
                    for (int q = 0; q < nq; ++q)
                        for (int kk = 0; kk < 2; ++kk)
                            tma_load_4d(sB + kk * 32768 + q * 16384, &mB, &b_full, kk * 64, g, t0 + q * kRows, b);
                    wait_bar(&b_full, bcnt++ & 1, status);
                    cur_b = b;
                    cur_c = c;
                    cur_g = g;
                }
                wait_bar(&x_ready[buf], (k >> 1) & 1, status);
                // this accumulator was last drained for tile k-2
                if (k >= 2) wait_bar(&acc_free[buf], ((k - 2) >> 1) & 1, status);
                fence_after_sync();
                for (int part = 0; part < 2; ++part)
                    for (int kk = 0; kk < sh.Q / 16; ++kk)
                        mma_ss(tmem + buf * 64, smem_desc_sw128(smem_u32(sB) + kk * 2048, 32768, 1024),
                               smem_desc_sw128(smem_u32(part ? sXlo : sX) + kk * 2048, 16, 1024), id,
                               part > 0 || kk > 0);
                mma_commit(&done[buf]);
            }
            // nothing this CTA issued is in flight when it leaves
            const int n = t_end - t_beg;
            for (int k = max(0, n - 2); k < n; ++k) wait_bar(&done[k & 1], (k >> 1) & 1, status);
        }
        __syncwarp();
    } else {
        const int wq = warp & 3, half = warp >> 2;
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        // S^T of tile k in tensor memory: lane n, column p; warpgroup `half` writes p in [32 half, 32 half + 32)
        auto drain = [&](int t, int k) {
            int b, c, h;
            tile(t, b, c, h);
            const int buf = k & 1, n = wq * 32 + lane;
            wait_bar(&done[buf], (k >> 1) & 1, status);
            fence_after_sync();
            float *Sp = S + (((size_t)b * sh.nc + c) * sh.H + h) * (size_t)(64 * 128);
#pragma unroll
            for (int q0 = 0; q0 < 32; q0 += 16) {
                uint32_t u[16];
                tmem_ld16(tmem + buf * 64 + half * 32 + q0 + lane_base, u);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) Sp[(size_t)(half * 32 + q0 + e) * 128 + n] = __uint_as_float(u[e]);
            }
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_free[buf]);
        };
        for (int t = t_beg, k = 0; t < t_end; ++t, ++k) {
            int b, c, h;
            tile(t, b, c, h);
            const int buf = k & 1, len = min(sh.Q, sh.T - c * sh.Q);
            uint8_t *sX = smem + cs::kOffX + buf * 32768, *sXlo = smem + cs::kOffXlo + buf * 32768;
            // weight each token row in place (high part) and into the low part; the weight's prefix sums
            // are loaded while x is on its way
            const float *sc = s + (((size_t)b * sh.H + h) * sh.nc + c) * sh.Q;
            const int i = tid;  // token row of the chunk
            const float si = (i < len) ? sc[i] : 0.f, send = sc[sh.Q - 1];
            wait_bar(&x_full[buf], (k >> 1) & 1, status);
            if (i < sh.Q) {
                const float w = (i < len) ? ex2((from_start ? si : send - si) * kLog2e) : 0.f;
                uint8_t *row = sX + (i >> 7) * 16384, *rowlo = sXlo + (i >> 7) * 16384;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = swz(i & 127, kk);
                    const uint4 v = *reinterpret_cast<const uint4 *>(row + off);
                    const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float a0 = bf16lo(vv[e]) * w, a1 = bf16hi(vv[e]) * w;
                        hi[e] = pack_bf16x2(a0, a1);
                        lo[e] = pack_lo(a0, a1, hi[e]);
                    }
                    *reinterpret_cast<uint4 *>(row + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    *reinterpret_cast<uint4 *>(rowlo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                }
            }
            fence_view_async_shared();
            __syncwarp();
            if (lane == 0) mbar_arrive(&x_ready[buf]);
            // the previous tile's state, while this one's product runs
            if (k >= 1) drain(t - 1, k - 1);
        }
        drain(t_end - 1, t_end - 1 - t_beg);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
bool scan_tc_supported(const Shape &sh, int dtype) {
    return dtype == SSD_BF16 && sh.P == 64 && (sh.N == 64 || sh.N == 128) && (sh.Q == 128 || sh.Q == 256) &&
           sh.batch <= 65535 && sh.H <= 65535;
}

int sm_count() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess || sms <= 0)
        sms = 148;
    return sms;
}

// CTAs of the head-summing scans (one per SM, at most kBwdSumMaxCtas, at most one per tile); the scans and the
// sum over their partial results take the same number
int head_sum_ctas(const Shape &sh) {
    const long long tiles = (long long)sh.batch * sh.nc * (sh.Q / kRows) * sh.H;
    return (int)std::min<long long>(tiles, std::min(sm_count(), kBwdSumMaxCtas));
}

// One masked scan.  R, K, V: bf16 [batch][T][heads or groups][KD, KD, W]; *_head: 1 = per head, 0 = per
// group.  St, st_kw, D, out as for the CUDA-core scan; out bf16 (dx) or fp32.  With `part` given the
// per-head terms are summed over each group's heads instead (out unused): part receives the CTAs'
// partial sums, dotp each head's rows dotted with the rows of dotv (see masked_scan_tc_kernel, kSum).
cudaError_t launch_masked_scan_tc(const void *R, int r_head, const void *K, int k_head, const void *V, int v_head,
                                  int KD, int W, bool anti, const float *St, int st_kw, const float *D, void *out,
                                  bool out_bf16, const float *s, int *status, const Shape &sh, cudaStream_t st,
                                  const void *dotv, float *dotp, float *part) {
    auto dims = [&](int head, int d, uint64_t *dm, uint64_t *sb) {
        const int n = head ? sh.H : sh.G;
        dm[0] = (uint64_t)d;
        dm[1] = (uint64_t)n;
        dm[2] = (uint64_t)sh.T;
        dm[3] = (uint64_t)sh.batch;
        sb[0] = (uint64_t)d * 2;
        sb[1] = (uint64_t)n * d * 2;
        sb[2] = (uint64_t)sh.T * n * d * 2;
    };
    const uint32_t box[4] = {64, 1, kRows, 1};
    CUtensorMap mR, mK, mV;
    uint64_t dm[4], sb[3];
    dims(r_head, KD, dm, sb);
    if (!make_map_bf16(&mR, R, 4, dm, sb, box)) return cudaErrorInvalidValue;
    dims(k_head, KD, dm, sb);
    if (!make_map_bf16(&mK, K, 4, dm, sb, box)) return cudaErrorInvalidValue;
    dims(v_head, W, dm, sb);
    if (!make_map_bf16(&mV, V, 4, dm, sb, box)) return cudaErrorInvalidValue;
    Args a;
    a.s = s;
    a.St = St;
    a.st_kw = st_kw;
    a.D = D;
    a.V = static_cast<const __nv_bfloat16 *>(V);
    a.v_head = v_head;
    a.out = out;
    a.status = status;
    a.sh = sh;
    a.dotv = static_cast<const __nv_bfloat16 *>(dotv);
    a.dotp = dotp;
    a.part = part;
    const bool sum = part != nullptr;
    if (sum && (out_bf16 || !dotv || !dotp)) return cudaErrorInvalidValue;
    void (*k)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const Args, int, int, int) = nullptr;
#define SSD_SCAN_TC_CASE(KDv, Wv, AN, OB, SP, SU)                                                  \
    if (KD == KDv && W == Wv && anti == AN && out_bf16 == OB && sum == SU) \
        k = masked_scan_tc_kernel<KDv, Wv, AN, OB, SP, SU>;
    SSD_SCAN_TC_CASE(128, 64, true, true, false, false)   // dx at N = 128
    SSD_SCAN_TC_CASE(64, 64, true, true, false, false)    // dx at N = 64
    SSD_SCAN_TC_CASE(64, 128, true, false, true, false)   // dB^(h) at N = 128
    SSD_SCAN_TC_CASE(64, 64, true, false, true, false)    // dB^(h) at N = 64
    SSD_SCAN_TC_CASE(64, 128, false, false, true, false)  // dC^(h) at N = 128
    SSD_SCAN_TC_CASE(64, 64, false, false, true, false)   // dC^(h) at N = 64
    SSD_SCAN_TC_CASE(64, 128, true, false, true, true)    // dB head sums at N = 128
    SSD_SCAN_TC_CASE(64, 64, true, false, true, true)     // dB head sums at N = 64
    SSD_SCAN_TC_CASE(64, 128, false, false, true, true)   // dC head sums at N = 128
    SSD_SCAN_TC_CASE(64, 64, false, false, true, true)    // dC head sums at N = 64
#undef SSD_SCAN_TC_CASE
    if (!k) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM, each taking every grid-th (chunk, block, head) tile, or (head sums) a
    // contiguous run of them
    const int tiles = sh.batch * sh.nc * (sh.Q / kRows) * sh.H;
    const int grid = sum ? head_sum_ctas(sh) : min(tiles, sm_count());
    if (sum) {
        TilePart tp;
        tp.init(sh, anti, grid);
        if (tp.tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
        tp.ranges(&a.tr);
    }
    k<<<grid, kThreads, kSmemBytes, st>>>(mR, mK, mV, a, r_head, k_head, v_head);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// The sums over each group's heads from the head-summing scans' partial results.  One block per (32
// tokens, group, batch) (32 tokens never straddle a 128-row block): it finds which CTAs took part of the
// tokens' (chunk, block, group) for dB and for dC (one candidate CTA per thread, from the scans' run
// table), adds their partial rows in CTA order, writes dB and dC, and each of the
// group's heads' dsigma_t = C_t . dC^(h)_t - B_t . dB^(h)_t from the scans' half-row dot products.
// 256 threads; each thread takes 4 consecutive n of a row.
// ---------------------------------------------------------------------------
constexpr int kRedTok = 32;

__global__ void __launch_bounds__(256) head_sum_reduce_kernel(const float *__restrict__ partB,
                                                              const float *__restrict__ dotB,
                                                              const float *__restrict__ partC,
                                                              const float *__restrict__ dotC,
                                                              const __grid_constant__ TileRanges rB,
                                                              const __grid_constant__ TileRanges rC,
                                                              __nv_bfloat16 *__restrict__ dB,
                                                              __nv_bfloat16 *__restrict__ dC, float *__restrict__ dsig,
                                                              Shape sh) {
    static_assert(kBwdSumMaxCtas <= 256, "one candidate CTA per thread");
    __shared__ int slots[2][kBwdSumMaxCtas];  // partial-sum slots of the contributing CTAs, in CTA order
    __shared__ int nslot[2];
    const int tid = threadIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tb = blockIdx.x * kRedTok;  // first token
    const int c = tb / sh.Q, rb = (tb - c * sh.Q) / kRows, lr0 = tb - c * sh.Q - rb * kRows;
    const int hpg = sh.heads_per_group;
    const long long blk = ((long long)b * sh.nc + c) * (sh.Q / kRows) + rb;
    const long long key = blk * sh.G + g, k0 = blk * sh.H + (long long)g * hpg;
    // CTA tid contributes when its run holds a head of the key (tiles k0 .. k0 + hpg - 1)
    for (int w = 0; w < 2; ++w) {
        const TileRanges &rg = w ? rC : rB;
        const int i = tid;
        const bool take = i < rg.ncta && max((long long)rg.beg[i], k0) < min((long long)rg.beg[i + 1], k0 + hpg);
        // compact in CTA order: a block-wide prefix count over the candidates
        const unsigned bal = __ballot_sync(0xffffffffu, take);
        __shared__ int wcnt[8];
        if ((tid & 31) == 0) wcnt[tid >> 5] = __popc(bal);
        __syncthreads();
        int before = __popc(bal & ((1u << (tid & 31)) - 1u));
        for (int q = 0; q < (tid >> 5); ++q) before += wcnt[q];
        if (take) slots[w][before] = i + (int)key;
        if (tid == 0) {
            int n = 0;
            for (int q = 0; q < 8; ++q) n += wcnt[q];
            nslot[w] = n;
        }
        __syncthreads();
    }
    const int V = sh.N / 4;  // 4-vectors per row
    const int ntok = min(kRedTok, sh.T - tb);
    // this thread's items (row, 4-vector) tid, tid + 256, ...: every slot's loads for all of them go out
    // together
    constexpr int kItems = kRedTok * 64 / 256;  // N <= 256
    float4 sb[kItems], sc[kItems];
#pragma unroll
    for (int q = 0; q < kItems; ++q) sb[q] = sc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    auto gather = [&](const float *part, int w, float4 (&acc)[kItems]) {
        for (int k = 0; k < nslot[w]; ++k) {
            const float *base = part + ((size_t)slots[w][k] * kRows + lr0) * sh.N;
#pragma unroll
            for (int q = 0; q < kItems; ++q) {
                const int item = tid + 256 * q, r = item / V, v = item - r * V;
                if (r < ntok) {
                    const float4 x = *reinterpret_cast<const float4 *>(base + (size_t)r * sh.N + 4 * v);
                    acc[q].x += x.x;
                    acc[q].y += x.y;
                    acc[q].z += x.z;
                    acc[q].w += x.w;
                }
            }
        }
    };
    gather(partB, 0, sb);
    gather(partC, 1, sc);
#pragma unroll
    for (int q = 0; q < kItems; ++q) {
        const int item = tid + 256 * q, r = item / V, v = item - r * V;
        if (r >= ntok) continue;
        const size_t grow = (((size_t)b * sh.T + tb + r) * sh.G + g) * sh.N + 4 * v;  // row (b, t, g)
        const __nv_bfloat162 b0 = __floats2bfloat162_rn(sb[q].x, sb[q].y), b1 = __floats2bfloat162_rn(sb[q].z, sb[q].w);
        const __nv_bfloat162 c0 = __floats2bfloat162_rn(sc[q].x, sc[q].y), c1 = __floats2bfloat162_rn(sc[q].z, sc[q].w);
        uint2 ub, uc;
        ub.x = *reinterpret_cast<const uint32_t *>(&b0);
        ub.y = *reinterpret_cast<const uint32_t *>(&b1);
        uc.x = *reinterpret_cast<const uint32_t *>(&c0);
        uc.y = *reinterpret_cast<const uint32_t *>(&c1);
        *reinterpret_cast<uint2 *>(dB + grow) = ub;
        *reinterpret_cast<uint2 *>(dC + grow) = uc;
    }
    // dsigma: a warp per head, a lane per token
    const int lane = tid & 31;
#pragma unroll 4
    for (int hh = tid >> 5; hh < hpg; hh += 8) {
        if (lane >= ntok) continue;
        const size_t at = ((size_t)b * sh.H + g * hpg + hh) * sh.T + tb + lane;
        const float2 db = *reinterpret_cast<const float2 *>(dotB + 2 * at);
        const float2 dc = *reinterpret_cast<const float2 *>(dotC + 2 * at);
        dsig[at] = (dc.x + dc.y) - (db.x + db.y);
    }
}

cudaError_t launch_head_sum_reduce(const float *partB, const float *dotB, const float *partC, const float *dotC,
                                   void *dB, void *dC, float *dsig, const Shape &sh, cudaStream_t st) {
    if (sh.N % 4 != 0 || sh.N > 256 || sh.G > 65535 || sh.batch > 65535) return cudaErrorInvalidValue;
    const int n = head_sum_ctas(sh);
    TilePart pb, pc;
    pb.init(sh, true, n);
    pc.init(sh, false, n);
    if (pb.tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
    TileRanges rB, rC;
    pb.ranges(&rB);
    pc.ranges(&rC);
    const dim3 grid((unsigned)((sh.T + kRedTok - 1) / kRedTok), (unsigned)sh.G, (unsigned)sh.batch);
    head_sum_reduce_kernel<<<grid, 256, 0, st>>>(partB, dotB, partC, dotC, rB, rC, static_cast<__nv_bfloat16 *>(dB),
                                                 static_cast<__nv_bfloat16 *>(dC), dsig, sh);
    return cudaGetLastError();
}

bool chunk_state_tc_supported(const Shape &sh, int dtype) {
    return dtype == SSD_BF16 && sh.P == 64 && sh.N == 128 && (sh.Q == 128 || sh.Q == 256) && sh.batch <= 65535 &&
           sh.H <= 65535;
}

// S [batch][nc][H][64][128] = the chunk states of x (per head) against B (per group), weighted from the
// chunk's end, or from its start (from_start).
cudaError_t launch_chunk_state_tc(const void *x, const void *B, const float *s, float *S, bool from_start,
                                  int *status, const Shape &sh, cudaStream_t st) {
    const uint32_t box[4] = {64, 1, kRows, 1};
    CUtensorMap mX, mB;
    const uint64_t dx[4] = {64, (uint64_t)sh.H, (uint64_t)sh.T, (uint64_t)sh.batch};
    const uint64_t sx[3] = {128, (uint64_t)sh.H * 128, (uint64_t)sh.T * sh.H * 128};
    const uint64_t db[4] = {128, (uint64_t)sh.G, (uint64_t)sh.T, (uint64_t)sh.batch};
    const uint64_t sbb[3] = {256, (uint64_t)sh.G * 256, (uint64_t)sh.T * sh.G * 256};
    if (!make_map_bf16(&mX, x, 4, dx, sx, box) || !make_map_bf16(&mB, B, 4, db, sbb, box))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_state_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)cs::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int tiles = sh.nc * sh.H * sh.batch;
    const int grid = min(tiles, sm_count()), per_cta = (tiles + grid - 1) / grid;
    chunk_state_tc_kernel<<<grid, kThreads, cs::kSmemBytes, st>>>(mX, mB, s, S, status, sh, from_start ? 1 : 0,
                                                                   per_cta);
    return cudaGetLastError();
}

}  // namespace ssd
