// attention.cu -- gather attention over the drawn key/value blocks
// ("Accurate Block Attention", abstract, kernel sentence: key/value blocks
// much smaller than a tile are gathered into full tensor-core tiles; SIP
// sentence: each drawn block is re-weighted by 1/pi, here as +ln(1/pi) on
// its logits inside the online softmax).
//
// B200 design.  Neighbouring query blocks (rows 2p and 2p+1 of a head, a
// "pair") draw heavily overlapping lists, so they run together on one SM and
// share the gathers of the blocks both drew:
//
//   pair_union_kernel   lays the pair's two ascending lists out as one array
//                       of three ascending segments, [blocks both rows drew |
//                       row 0 only | row 1 only], with each row's base-2
//                       log-weights in the order that row walks them
//                       ([both | its own]; -inf up to the end of its last
//                       tile) and the position of the partial last key block.
//   gather_attn_kernel  persistent, one CTA per SM, one pair at a time.  Each
//                       row walks exactly its own blocks in 128-key tiles, so
//                       no tile holds a block the row did not draw; tiles that
//                       lie wholly inside the shared segment are gathered once
//                       (TMA boxes of one key block each, K and V) for both
//                       rows, later tiles per row.
//
// What bounds it is the per-row chain S(t) -> softmax(t) -> PV(t) -> S(t+1)
// (P replaces S in tensor memory): the softmax of a 128x128 tile is bound by
// issue slots and the ex2 unit, and the two rows' softmaxes overlap the other
// row's tensor-core work only partly.
//
// Warp roles (640 threads, five warpgroups; warpgroup 0 hands registers to
// the softmax warpgroups with setmaxnreg):
//   warp 0      TMA producer: Q of both rows, then K(t), V(t) into a ring;
//   warp 1      tensor-memory owner and tcgen05 MMA issuer:
//               S_s = Q_s K^T (fp32, 128 TMEM columns per row),
//               O_s += P_s V  (P_s read back from the columns S_s used);
//   warps 2-3   idle;
//   warps 4-19  softmax, eight warps per row s of the pair; a warp owns 16
//               query rows of its tensor-memory lane quarter and its two
//               half-warps split each row's 128 columns (two threads per
//               query): raw per-block maxima of the thread's 64 columns, the
//               row's tile maximum of s*log2(e)*S + log-weight (base 2) by one
//               shuffle, lazy running maximum (O is rescaled only when it
//               grows by more than 8), P in bf16 back into tensor memory,
//               final O / l to bf16 (each thread writes half of its row).
#include "kernels.cuh"

namespace abatt {

namespace {

constexpr int kAttnThreads = 640;   // warpgroup 0: TMA, MMA (+2 idle warps); 1-4: softmax
constexpr int kRegsControl = 56;     // registers per thread of warpgroup 0 after setmaxnreg
constexpr int kRegsSoftmax = 104;    // ... and of the four softmax warpgroups
#define kNegInf (-__int_as_float(0x7f800000))
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;
// exponent pairs of every eight that the softmax evaluates with the FMA-pipe
// polynomial (the others use ex2); balances the two pipes
#ifndef ABATT_ATTN_POLY_OF_8
#define ABATT_ATTN_POLY_OF_8 0
#endif
constexpr int kAttnPolyOf8 = ABATT_ATTN_POLY_OF_8;

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ============================== pair union ======================================
constexpr int kUnionThreads = 128;

// Entry j of a list is used if it is a block index and exceeds the previous
// entry (when that one is a block index itself).
__device__ __forceinline__ bool union_entry_ok(const int32_t *idx, int j, int k, int nK) {
    if (k < 0 || k >= nK) return false;
    if (j == 0) return true;
    const int prev = idx[j - 1];
    return prev < 0 || prev >= nK || prev < k;
}

__global__ void __launch_bounds__(kUnionThreads) pair_union_kernel(const PairArgs a) {
    // [W] membership bitmap of each row, then per word the exclusive prefix of
    // the three segment counts (both rows, row 0 only, row 1 only)
    extern __shared__ uint32_t sm_union[];
    __shared__ uint64_t wsum[kUnionThreads / 32];
    __shared__ int tail_pos_s;  // position of the partial last key block in the pair's array
    const bool ragged = a.ragged != 0;
    const int W = (a.nK + 31) >> 5;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t *bA = sm_union, *bB = sm_union + W;
    uint32_t *preB = sm_union + 2 * W, *preA = preB + W, *preC = preA + W;
    for (int64_t pr = blockIdx.x; pr < a.pairs; pr += gridDim.x) {
        __syncthreads();
        for (int w = tid; w < 2 * W; w += kUnionThreads) sm_union[w] = 0;
        if (tid == 0) tail_pos_s = -1;
        __syncthreads();
        int64_t rr[2];
        pair_rows(pr, a.nQ, &rr[0], &rr[1]);
        int L[2];
        bool bad = false;
        for (int s = 0; s < 2; ++s) {
            L[s] = rr[s] >= 0 ? min(max(a.counts[rr[s]], 0), a.capacity) : 0;
            const int32_t *idx = a.idx + (rr[s] >= 0 ? rr[s] : 0) * (int64_t)a.capacity;
            uint32_t *b = s ? bB : bA;
            for (int j = tid; j < L[s]; j += kUnionThreads) {
                const int k = idx[j];
                if (!union_entry_ok(idx, j, k, a.nK)) { bad = true; continue; }
                atomicOr(&b[k >> 5], 1u << (k & 31));
            }
        }
        if (__syncthreads_or(bad) && tid == 0) raise_flag(a.status, ABATT_DEVFLAG_BADLIST);
        // exclusive prefix of the three popcounts per word, packed 21 bits
        // each into one 64-bit scan: each thread owns a contiguous run of words
        const int per = (W + kUnionThreads - 1) / kUnionThreads;
        const int w0 = min(W, tid * per), w1 = min(W, w0 + per);
        auto counts3 = [&](int w) -> uint64_t {
            const uint32_t x = bA[w], y = bB[w];
            return (uint64_t)__popc(x & y) | ((uint64_t)__popc(x & ~y) << 21) |
                   ((uint64_t)__popc(y & ~x) << 42);
        };
        uint64_t cnt = 0;
        for (int w = w0; w < w1; ++w) cnt += counts3(w);
        uint64_t x = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[warp] = x;
        __syncthreads();
        uint64_t run = x - cnt, total = 0;
        for (int w = 0; w < kUnionThreads / 32; ++w) {
            if (w < warp) run += wsum[w];
            total += wsum[w];
        }
        constexpr uint64_t kM21 = (1u << 21) - 1u;
        for (int w = w0; w < w1; ++w) {
            preB[w] = (uint32_t)(run & kM21);
            preA[w] = (uint32_t)((run >> 21) & kM21);
            preC[w] = (uint32_t)(run >> 42);
            run += counts3(w);
        }
        const int nb = (int)(total & kM21), na = (int)((total >> 21) & kM21), nc = (int)(total >> 42);
        __syncthreads();
        int32_t *ub = a.ublk + pr * (int64_t)a.cap_u;
        // union layout: [both rows | row 0 only | row 1 only], each ascending
        for (int w = tid; w < W; w += kUnionThreads) {
            const uint32_t xa = bA[w], xb = bB[w];
            const uint32_t seg[3] = {xa & xb, xa & ~xb, xb & ~xa};
            const int base[3] = {(int)preB[w], nb + (int)preA[w], nb + na + (int)preC[w]};
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                int pos = base[q];
                for (uint32_t mu = seg[q]; mu; mu &= mu - 1) {
                    const int k = w * 32 + __ffs(mu) - 1;
                    if (pos < a.cap_u) ub[pos] = k;
                    if (ragged && k == a.nK - 1) tail_pos_s = pos;
                    ++pos;
                }
            }
        }
        // each valid drawn entry writes its row's base-2 log-weight at its index
        // in the row's sequence (row 0: [both | row 0 only] = positions 0..;
        // row 1: [both | row 1 only], its own segment na positions earlier)
        float *uw = a.ulw + pr * 2 * (int64_t)a.cap_w;
        for (int s = 0; s < 2; ++s) {
            const int32_t *idx = a.idx + (rr[s] >= 0 ? rr[s] : 0) * (int64_t)a.capacity;
            const float *lw = a.logw + (rr[s] >= 0 ? rr[s] : 0) * (int64_t)a.capacity;
            for (int j = tid; j < L[s]; j += kUnionThreads) {
                const int k = idx[j];
                if (!union_entry_ok(idx, j, k, a.nK)) continue;
                const int w = k >> 5;
                const uint32_t below = (1u << (k & 31)) - 1u;
                const uint32_t xa = bA[w], xb = bB[w];
                int pos;
                if ((xa & xb) >> (k & 31) & 1u) pos = (int)preB[w] + __popc(xa & xb & below);
                else if (s == 0) pos = nb + (int)preA[w] + __popc(xa & ~xb & below);
                else pos = nb + (int)preC[w] + __popc(xb & ~xa & below);
                if (pos < a.cap_u) uw[s * a.cap_w + pos] = lw[j] * kLog2e;
            }
            // -inf after the sequence up to the end of its last tile: the
            // attention kernel reads whole tiles of weights
            const int U = rr[s] >= 0 ? (s == 0 ? nb + na : nb + nc) : 0;
            const int Upad = (U + a.bpt - 1) / a.bpt * a.bpt;
            if (tid < Upad - U && U + tid < a.cap_w) uw[s * a.cap_w + U + tid] = kNegInf;
        }
        __syncthreads();  // tail_pos_s is written
        if (tid == 0) {
            a.useg[pr * 4 + 0] = nb;
            a.useg[pr * 4 + 1] = na;
            a.useg[pr * 4 + 2] = nc;
            a.useg[pr * 4 + 3] = tail_pos_s;
        }
    }
}

// ============================== attention ======================================
template <int D>
struct AttnCfg {
    static constexpr int CH = D / 64;
    static constexpr uint32_t TILE = 128u * D * 2u;
    static constexpr int ST = D == 128 ? 5 : 12;  // K/V ring stages (Q tiles + ring <= 225 KB)
    static constexpr size_t SMEM = (size_t)(2 + ST) * TILE + 1024;
};

// The tile schedule of one pair.  Row s walks its sequence (row 0: [both |
// row 0 only], row 1: [both | row 1 only]) in tiles of BPT blocks: n[s]
// tiles.  The first tb tiles lie wholly inside the shared segment and are
// gathered once for both rows; later tiles are gathered per row.  Gathers
// ("groups", a K tile and a V tile each, ring slots 2g and 2g+1 after the
// pair's first slot) run in step order: shared tiles 0..tb-1, then for each
// step t >= tb row 0's tile (if t < n[0]) and row 1's tile (if t < n[1]).
struct PairPlan {
    int nb, na, L0, L1, n0, n1, tb, m, groups;
    __device__ __forceinline__ PairPlan(const int32_t *useg, int64_t pr, bool has1, int bpt) {
        nb = useg[pr * 4 + 0];
        na = useg[pr * 4 + 1];
        const int nc = useg[pr * 4 + 2];
        L0 = nb + na;
        L1 = has1 ? nb + nc : 0;
        n0 = (L0 + bpt - 1) / bpt;
        n1 = (L1 + bpt - 1) / bpt;
        tb = has1 ? nb / bpt : 0;
        m = max(0, min(n0, n1) - tb);
        groups = n0 + n1 - tb;
    }
    __device__ __forceinline__ int L(int s) const { return s ? L1 : L0; }
    __device__ __forceinline__ int n(int s) const { return s ? n1 : n0; }
    // gather group of row s's tile t
    __device__ __forceinline__ int group(int s, int t) const {
        if (t < tb) return t;
        const int d = t - tb;
        return d < m ? tb + 2 * d + s : tb + 2 * m + (d - m);
    }
    // row (-1: shared) and tile of gather group g
    __device__ __forceinline__ void tile_of(int g, int *s, int *t) const {
        if (g < tb) { *s = -1; *t = g; return; }
        const int r = g - tb;
        if (r < 2 * m) { *s = r & 1; *t = tb + (r >> 1); return; }
        *s = n0 > n1 ? 0 : 1;
        *t = tb + m + (r - 2 * m);
    }
    // entry e of row s's sequence -> position in the pair's block array
    __device__ __forceinline__ int pos(int s, int e) const { return (s == 0 || e < nb) ? e : e + na; }
};

template <int D, int BK, bool KFOLD>
__global__ void __launch_bounds__(kAttnThreads, 1)
    gather_attn_kernel(const __grid_constant__ AttnMaps maps, const AttnArgs a) {
    using Cfg = AttnCfg<D>;
    constexpr int CH = Cfg::CH;
    constexpr uint32_t TILE = Cfg::TILE;
    constexpr int ST = Cfg::ST;
    constexpr int BPT = 128 / BK;
    constexpr uint32_t BLK = (uint32_t)BK * D * 2;  // bytes of one gathered block
    constexpr uint32_t TMEM_COLS = 512;             // S0 | S1 | O0 | O1

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sQ = smem;                // [2][TILE]
    uint8_t *sRing = smem + 2 * TILE;  // [ST][TILE]

    __shared__ __align__(8) uint64_t bar_qf[2], bar_qe[2];
    __shared__ __align__(8) uint64_t bar_kvf[ST], bar_kve[ST];
    __shared__ __align__(8) uint64_t bar_sf[2], bar_pf[2], bar_of[2], bar_oe[2];
    __shared__ __align__(8) uint64_t bar_drain;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;

    __shared__ int skip_s;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // a bounded wait elsewhere already gave up: start no more work.  One read,
    // shared by the whole CTA, so every role takes the same decision
    if (threadIdx.x == 0)
        skip_s = a.hdr && (*reinterpret_cast<volatile uint32_t *>(&a.hdr->status) & ABATT_DEVFLAG_TIMEOUT);
    __syncthreads();
    if (skip_s) return;
    const WaitCtx wc{&abort_s, a.hdr, a.wait_ns};

    if (threadIdx.x == 0) {
        abort_s = 0;
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar_qf[s], 1);
            mbar_init(&bar_qe[s], 1);
            mbar_init(&bar_sf[s], 1);
            mbar_init(&bar_pf[s], 8);
            mbar_init(&bar_of[s], 1);
            mbar_init(&bar_oe[s], 8);
        }
        for (int s = 0; s < ST; ++s) {
            mbar_init(&bar_kvf[s], 1);
            mbar_init(&bar_kve[s], 1);
        }
        mbar_init(&bar_drain, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_s, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;

    uint32_t ring_issued = 0;         // producer: ring loads issued (for the drain)
    uint32_t q_issued[2] = {0, 0};    // producer: Q loads issued per row slot (for the drain)

    if (warp == 0) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
        // ================================ TMA producer ================================
        // The whole warp: lane 0 owns the barriers; lane k < 128/Bk gathers
        // block k of each tile, its index prefetched one tile ahead.
        if (lane == 0) {
            tma_prefetch_desc(&maps.q);
            tma_prefetch_desc(&maps.k);
            tma_prefetch_desc(&maps.v);
        }
        uint32_t q_loads[2] = {0, 0};
        uint32_t rp = 0;
        bool ok = true;
        for (int64_t pr = blockIdx.x; ok && pr < a.pairs; pr += gridDim.x) {
            int64_t rr[2];
            pair_rows(pr, a.nQ, &rr[0], &rr[1]);
            const PairPlan P(a.useg, pr, rr[1] >= 0, BPT);
            if (P.groups == 0) continue;
            const int hd = (int)(rr[0] / a.nQ);
            const int bat = hd / a.st.H, hed = hd % a.st.H;  // batch element and head
            const int32_t *ub = a.ublk + pr * (int64_t)a.cap_u;
            // block index of this lane in gather group g (-1: empty slot)
            auto blk_of = [&](int g) -> int {
                if (g >= P.groups || lane >= BPT) return -1;
                int s, t;
                P.tile_of(g, &s, &t);
                const int sr = s < 0 ? 0 : s, e = t * BPT + lane;
                return e < P.L(sr) ? __ldg(ub + P.pos(sr, e)) : -1;
            };
            int nxt = blk_of(0);
            if (lane == 0) {
                for (int s = 0; s < 2; ++s) {
                    const int64_t row = rr[s];
                    if (row < 0 || P.n(s) == 0) continue;
                    if (q_loads[s] > 0 && !mbar_wait(&bar_qe[s], (q_loads[s] - 1) & 1, wc, 0x202)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bar_qf[s], TILE);
                    const int i = (int)(row % a.nQ);
                    for (int c = 0; c < CH; ++c)
                        tma_load_4d(sQ + s * TILE + c * 16384, &maps.q, &bar_qf[s], c * 64, i * 128, hed, bat);
                    ++q_loads[s];
                    q_issued[s] = q_loads[s];
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            for (int g = 0; ok && g < P.groups; ++g) {
                if (a.stall && rp >= 2) {  // test hook: no copy after the CTA's first K/V tile pair
                    ok = false;
                    break;
                }
                const int blk = nxt;
                nxt = blk_of(g + 1);
                for (int kv = 0; kv < 2; ++kv) {  // K then V of the group
                    const int stg = rp % ST;
                    if (lane == 0) {
                        if (rp >= ST && !mbar_wait(&bar_kve[stg], ((rp / ST) - 1) & 1, wc, 0x201)) ok = false;
                        if (ok) mbar_arrive_expect_tx(&bar_kvf[stg], TILE);
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    if (lane < BPT) {
                        uint8_t *dst = sRing + stg * TILE;
                        const bool valid = blk >= 0;
                        if (kv == 0) {
                            if (KFOLD) {
                                // a box of Bk/8 groups of 8 rows, all head-dim chunks
                                const int gy = valid ? bat * a.kf_gb + blk * (BK / 8) : 0x7fffff00;
                                tma_load_5d(dst + lane * BLK, &maps.k, &bar_kvf[stg], 0, 0, 0, gy,
                                            bat * a.kf_zb + hed);
                            } else {
                                const int y = valid ? blk * BK : a.nK * BK;
                                for (int c = 0; c < CH; ++c)
                                    tma_load_4d(dst + c * 16384 + lane * BK * 128, &maps.k, &bar_kvf[stg],
                                                c * 64, y, hed, bat);
                            }
                        } else {
                            const int y = valid ? blk * BK : a.nK * BK;
                            tma_load_5d(dst + lane * BLK, &maps.v, &bar_kvf[stg], 0, y, 0, hed, bat);
                        }
                    }
                    ++rp;
                    if (lane == 0) ring_issued = rp;
                }
            }
        }
    } else if (warp == 1) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
        // ================================ MMA issuer ==================================
        // The whole warp runs the schedule, so its control flow and the
        // descriptors stay warp-uniform; one elected lane issues each tcgen05
        // instruction.
        constexpr uint32_t idesc_s = idesc_bf16(128, 128);
        constexpr uint32_t idesc_o = idesc_bf16(128, D, /*b_mn_major=*/true);
        uint32_t rp = 0;  // ring position of K(t); V(t) is rp+1
        uint32_t q_uses[2] = {0, 0}, pv_ops[2] = {0, 0}, o_items[2] = {0, 0};
        bool ok = true;
        const uint32_t q_addr0 = smem_u32(sQ), ring_addr = smem_u32(sRing);  // < 256 KB: the
        // 14-bit address field of a descriptor never carries into the next field
        auto wait_all = [&](uint64_t *bar, uint32_t parity, uint32_t site) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc, site));
        };
        // K(t) / V(t) have landed (called before the waits that gate issue)
        auto wait_kv = [&](uint32_t pos, uint32_t site) -> bool {
            return wait_all(&bar_kvf[pos % ST], (pos / ST) & 1, site);
        };
        auto op_s = [&](int s, uint32_t kpos, bool release, bool last) {
            const int stg = kpos % ST;
            tc_fence_after();
            // descriptors built once per op; each k-step adds its byte offset / 16
            const uint64_t qd = sdesc_sw128(q_addr0 + s * TILE, 16, 1024);
            const uint64_t kd = sdesc_sw128(ring_addr + stg * TILE, 16, KFOLD ? CH * 1024 : 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t qoff = (kk >> 2) * 16384 + (kk & 3) * 32;
                const uint32_t koff =
                    KFOLD ? (kk >> 2) * 1024 + (kk & 3) * 32 : (kk >> 2) * 16384 + (kk & 3) * 32;
                umma_ss_w(tmem + s * 128, qd + (qoff >> 4), kd + (koff >> 4), idesc_s, kk > 0);
            }
            if (release) umma_commit_w(&bar_kve[stg]);
            umma_commit_w(&bar_sf[s]);
            if (last) umma_commit_w(&bar_qe[s]);
        };
        auto op_pv = [&](int s, uint32_t vpos, int t, bool release, bool last) -> bool {
            if (t == 0 && o_items[s] > 0 && !wait_all(&bar_oe[s], (o_items[s] - 1) & 1, 0x205))
                return false;
            if (!wait_all(&bar_pf[s], pv_ops[s] & 1, 0x204)) return false;
            const int stg = vpos % ST;
            tc_fence_after();
            const uint64_t vd = sdesc_sw128(ring_addr + stg * TILE, BK * 128, 1024);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t boff = (uint32_t)((16 * j) / BK) * BLK + (uint32_t)((16 * j) % BK) * 128;
                umma_ts_w(tmem + 256 + s * 128, tmem + s * 128 + j * 8, vd + (boff >> 4), idesc_o,
                               (t > 0 || j > 0) ? 1u : 0u);
            }
            if (release) umma_commit_w(&bar_kve[stg]);
            if (last) {
                umma_commit_w(&bar_of[s]);
                ++o_items[s];
            }
            ++pv_ops[s];
            return true;
        };
        for (int64_t pr = blockIdx.x; ok && pr < a.pairs; pr += gridDim.x) {
            int64_t rr[2];
            pair_rows(pr, a.nQ, &rr[0], &rr[1]);
            const PairPlan P(a.useg, pr, rr[1] >= 0, BPT);
            if (P.groups == 0) continue;
            for (int s = 0; ok && s < 2; ++s) {
                if (P.n(s) == 0) continue;
                if (!wait_all(&bar_qf[s], q_uses[s] & 1, 0x207)) ok = false;
                ++q_uses[s];
            }
            const uint32_t base = rp;
            auto kpos = [&](int s, int t) -> uint32_t { return base + 2u * (uint32_t)P.group(s, t); };
            // a shared tile's slots are freed by row 1's MMA (issued after row 0's)
            auto frees = [&](int s, int t) -> bool { return t >= P.tb || s == 1; };
            // issue order per step t: PV0(t) S0(t+1) PV1(t) S1(t+1).  Each row's
            // chain is softmax(t) -> PV(t) -> S(t+1) (S(t+1) overwrites the P(t)
            // that PV(t) reads; tcgen05 MMAs of one thread run in issue order).
            // Waits for K/V data sit before the wait on P, so once P is ready
            // nothing else delays the two MMAs of its row.
            for (int s = 0; ok && s < 2; ++s) {
                if (P.n(s) == 0) continue;
                if (!wait_kv(kpos(s, 0), 0x203)) { ok = false; break; }
                op_s(s, kpos(s, 0), frees(s, 0), P.n(s) == 1);
            }
            const int T = max(P.n0, P.n1);
            for (int t = 0; ok && t < T; ++t) {
                for (int s = 0; s < 2; ++s) {
                    if (t >= P.n(s)) continue;
                    const bool more = t + 1 < P.n(s);
                    const uint32_t vp = kpos(s, t) + 1;
                    if (!wait_kv(vp, 0x206) || (more && !wait_kv(kpos(s, t + 1), 0x203))) { ok = false; break; }
                    if (!op_pv(s, vp, t, frees(s, t), !more)) { ok = false; break; }
                    if (more) op_s(s, kpos(s, t + 1), frees(s, t + 1), t + 2 == P.n(s));
                }
            }
            rp = base + 2u * (uint32_t)P.groups;
        }
    } else if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));  // idle
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        // ================================ softmax =====================================
        // Eight warps per row of the pair.  A warp owns 16 query rows (TMEM
        // lanes) of its lane quarter; the two half-warps split each row's
        // columns, so a row's maximum and sum need one shuffle, not a barrier.
        constexpr int HB = BPT >= 2 ? BPT / 2 : 1;  // blocks (or block parts) per column half
        const int sw = warp - 4;
        const int s = sw >> 3;              // row of the pair
        const int sub = (sw >> 2) & 1;      // 16-lane half of the lane quarter
        const int wq = warp & 3;            // tensor-memory lane quarter
        const int hh = lane >> 4;           // column half of each tile
        const int r = wq * 32 + sub * 16 + (lane & 15);  // query row within the block == TMEM lane
        const uint32_t t_lane = (uint32_t)(wq * 32 + sub * 16) << 16;
        const uint32_t s_col = tmem + t_lane + s * 128;
        const uint32_t o_col = tmem + t_lane + 256 + s * 128;
        uint32_t s_uses = 0, o_uses = 0;
        bool ok = true;
        for (int64_t pr = blockIdx.x; ok && pr < a.pairs; pr += gridDim.x) {
            int64_t rr[2];
            pair_rows(pr, a.nQ, &rr[0], &rr[1]);
            const int64_t row = rr[s];
            if (row < 0) continue;  // the pair's second row does not exist
            const PairPlan P(a.useg, pr, rr[1] >= 0, BPT);
            const int U = P.L(s), n = P.n(s);
            const int i = (int)(row % a.nQ), hd = (int)(row / a.nQ);
            const int nrows = min(128, a.N - i * 128);
            const int64_t tok = (int64_t)hd * a.N + (int64_t)i * 128 + r;
            const float *lw = a.ulw + (pr * 2 + s) * (int64_t)a.cap_w;
            float m_run = kNegInf, l = 0.0f;
            // entry of this row's sequence that holds the partial last key
            // block (-1: none): its keys past N are masked
            const int tp = a.useg[pr * 4 + 3];
            const int etail = tp < 0 ? -1
                              : s == 0 ? (tp < P.nb + P.na ? tp : -1)
                                       : (tp < P.nb ? tp : (tp >= P.nb + P.na ? tp - P.na : -1));
            const int tail_keep = a.N - (a.nK - 1) * BK;
            // base-2 log-weights of this half's blocks for the next tile (the
            // row's sequence, -inf past its end), one vector load one tile ahead,
            // first read at that tile (its latency hides behind the current tile)
            float nw[HB];
            auto load_meta = [&](int t) {
                const float *src = lw + t * BPT + (BPT >= 2 ? hh * HB : 0);
                if constexpr (HB == 4) {
                    const float4 q = __ldg(reinterpret_cast<const float4 *>(src));
                    nw[0] = q.x; nw[1] = q.y; nw[2] = q.z; nw[3] = q.w;
                } else if constexpr (HB == 2) {
                    const float2 q = __ldg(reinterpret_cast<const float2 *>(src));
                    nw[0] = q.x; nw[1] = q.y;
                } else {
                    nw[0] = __ldg(src);
                }
            };
            if (n > 0) load_meta(0);
            for (int t = 0; t < n; ++t) {
                float bias[HB];
#pragma unroll
                for (int k = 0; k < HB; ++k) bias[k] = nw[k];
                int tail_k = -1;
                {
                    const int et = etail - t * BPT;  // the tail block's slot in this tile
                    if (et >= 0 && et < BPT) {
                        const int k = BPT >= 2 ? et - hh * HB : 0;
                        if (k >= 0 && k < HB) tail_k = k;
                    }
                }
                if (t + 1 < n) load_meta(t + 1);
                const bool masked = tail_k >= 0;
                // warp-uniform outcome: the lanes go on to warp-collective tcgen05 loads
                if (!__all_sync(0xffffffffu, mbar_wait(&bar_sf[s], s_uses & 1, wc, 0x208))) { ok = false; break; }
                ++s_uses;
                tc_fence_after();
                uint32_t v[2][32];
#pragma unroll
                for (int c = 0; c < 2; ++c) tmem_ld32_split<64>(s_col + c * 32, v[c]);
                tmem_wait_ld();
                // column (within the tile) of v[c][j]: 64*hh + 32*c + j; its block
                // slot within this half: (32c + j) / BK (or 0 for blocks wider
                // than a half); its key within the block: column % BK
                if (masked) {
#pragma unroll
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int col = hh * 64 + c * 32 + j;
                            const int k = BPT >= 2 ? (c * 32 + j) / BK : 0;
                            if (k == tail_k && col % BK >= tail_keep) v[c][j] = __float_as_uint(kNegInf);
                        }
                }
                // raw maximum of each block's columns in this half (a tree: short
                // dependency chains), then the half's maximum of scaled + weighted
                constexpr int VPB = 64 / HB;  // columns of one block (part) in this half
                float hm[HB];
#pragma unroll
                for (int k = 0; k < HB; ++k) {
                    float w[VPB];
#pragma unroll
                    for (int e = 0; e < VPB; ++e) {
                        const int col = k * VPB + e;  // 0..63 within the half
                        w[e] = __uint_as_float(v[col >> 5][col & 31]);
                    }
                    hm[k] = fmaf(max_tree<VPB>(w), a.scale_log2, bias[k]);
                }
                const float hmax = max_tree<HB>(hm);
                const float tmax = fmaxf(hmax, __shfl_xor_sync(0xffffffffu, hmax, 16));
                const bool need = tmax > m_run + kRescaleThreshold;
                const float m_use = need ? tmax : m_run;
                const float alpha = need ? ((m_run == kNegInf) ? 0.0f : ex2_approx(m_run - tmax)) : 1.0f;
                const float m_sub = (m_use == kNegInf) ? 0.0f : m_use;
#pragma unroll
                for (int k = 0; k < HB; ++k) bias[k] -= m_sub;  // now the exponent offset
                // exponents two at a time (packed fp32 FMA / add); a fixed share
                // of the pairs goes to the FMA-pipe polynomial, the rest to ex2
                const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
                float2 rs2[4];  // four independent partial row sums
#pragma unroll
                for (int u = 0; u < 4; ++u) rs2[u] = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        // columns j, j+1 lie in one key block (blocks are >= 16 wide)
                        const int k0 = BPT >= 2 ? (c * 32 + j) / BK : 0;
                        const float2 x = __ffma2_rn(make_float2(__uint_as_float(v[c][j]), __uint_as_float(v[c][j + 1])),
                                                    sc2, make_float2(bias[k0], bias[k0]));
                        float2 p;
                        if (((c * 16 + (j >> 1)) & 7) < kAttnPolyOf8) {
                            p = exp2_poly2<3>(x);
                        } else {
                            p.x = ex2_approx(x.x);
                            p.y = ex2_approx(x.y);
                        }
                        rs2[(j >> 1) & 3] = __fadd2_rn(rs2[(j >> 1) & 3], p);
                        pk[j >> 1] = pack_bf16x2(p.x, p.y);
                    }
                    // P (bf16 pairs) over the row's S: this half's keys 64*hh + 32c + 0..31
                    // go to packed columns 32*hh + 16c + 0..15; both halves of the warp
                    // finished reading S above
                    tmem_st16_split<32>(s_col + c * 16, pk);
                }
                // rescale this row's O (after P, so the scores are dead): the
                // commit that signalled S(t) covers the previous PV
                if (t > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
                    for (int c = 0; c < D / 64; ++c) {
                        uint32_t o[32];
                        const uint32_t oa = o_col + c * 32;
                        tmem_ld32_split<D / 2>(oa, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                        tmem_st32_split<D / 2>(oa, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_pf[s]);
                const float2 rs = __fadd2_rn(__fadd2_rn(rs2[0], rs2[1]), __fadd2_rn(rs2[2], rs2[3]));
                l = fmaf(l, alpha, rs.x + rs.y);
                m_run = m_use;
            }
            if (!ok) break;
            __nv_bfloat16 *orow = a.O + a.st.head_base(hd) + (int64_t)(i * 128 + r) * a.st.sT + hh * (D / 2);
            if (n == 0) {  // no block at all: O = 0, lse = -inf
                if (r < nrows) {
#pragma unroll
                    for (int q = 0; q < D / 16; ++q) reinterpret_cast<uint4 *>(orow)[q] = make_uint4(0, 0, 0, 0);
                    if (a.lse && hh == 0) a.lse[tok] = kNegInf;
                }
                continue;
            }
            // epilogue: the row sum is split over the two half-warps
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            if (!__all_sync(0xffffffffu, mbar_wait(&bar_of[s], o_uses & 1, wc, 0x209))) { ok = false; break; }
            ++o_uses;
            tc_fence_after();
            const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                uint32_t o[32];
                tmem_ld32_split<D / 2>(o_col + c * 32, o);
                tmem_wait_ld();
                if (r < nrows) {
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(o[j + 0]) * inv, __uint_as_float(o[j + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(o[j + 2]) * inv, __uint_as_float(o[j + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(o[j + 4]) * inv, __uint_as_float(o[j + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(o[j + 6]) * inv, __uint_as_float(o[j + 7]) * inv);
                        *reinterpret_cast<uint4 *>(orow + c * 32 + j) = w;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_oe[s]);
            if (a.lse && hh == 0 && r < nrows) a.lse[tok] = l > 0.0f ? (m_run + __log2f(l)) * kLn2 : kNegInf;
        }
        tc_fence_before();
    }

    // ================================ teardown ========================================
    __syncthreads();
    if (abort_s) {
        // let copies still in flight land before shared memory goes away
        if (warp == 0 && lane == 0) {
            for (uint32_t q = ring_issued > ST ? ring_issued - ST : 0; q < ring_issued; ++q) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&bar_kvf[q % ST], (q / ST) & 1) &&
                       globaltimer_ns() - t0 < a.wait_ns) {
                }
            }
            for (int s = 0; s < 2; ++s) {  // the last Q load of each row slot
                if (q_issued[s] == 0) continue;
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&bar_qf[s], (q_issued[s] - 1) & 1) && globaltimer_ns() - t0 < a.wait_ns) {
                }
            }
        }
        // and MMAs: a commit issued now arrives once all earlier MMAs are done
        if (warp == 1 && lane == 0) {
            umma_commit(&bar_drain);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&bar_drain, 0) && globaltimer_ns() - t0 < a.wait_ns) {
            }
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <int D, int BK, bool KF>
cudaError_t launch_attn_t(const AttnArgs &a, const AttnMaps &maps, int num_sms, cudaStream_t stream) {
    const size_t smem = AttnCfg<D>::SMEM;
    cudaError_t e = cudaFuncSetAttribute(gather_attn_kernel<D, BK, KF>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // setmaxnreg moves registers between warpgroups within the launch's
    // allocation: the compiled count must cover the split, else the
    // increase would never be granted
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, gather_attn_kernel<D, BK, KF>);
    if (e != cudaSuccess) return e;
    if ((int64_t)fa.numRegs * kAttnThreads < 128 * kRegsControl + (kAttnThreads - 128) * kRegsSoftmax)
        return cudaErrorInvalidConfiguration;
    const int grid = (int)(a.pairs < num_sms ? a.pairs : num_sms);
    gather_attn_kernel<D, BK, KF><<<grid, kAttnThreads, smem, stream>>>(maps, a);
    return cudaGetLastError();
}

template <int D, int BK>
cudaError_t launch_attn_k(const AttnArgs &a, const AttnMaps &maps, int num_sms, cudaStream_t stream) {
    return a.k_fold ? launch_attn_t<D, BK, true>(a, maps, num_sms, stream)
                    : launch_attn_t<D, BK, false>(a, maps, num_sms, stream);
}

template <int D>
cudaError_t launch_attn_d(const AttnArgs &a, const AttnMaps &maps, int num_sms, cudaStream_t stream) {
    switch (a.Bk) {
        case 16: return launch_attn_k<D, 16>(a, maps, num_sms, stream);
        case 32: return launch_attn_k<D, 32>(a, maps, num_sms, stream);
        case 64: return launch_attn_k<D, 64>(a, maps, num_sms, stream);
        case 128: return launch_attn_k<D, 128>(a, maps, num_sms, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_pair_union(const PairArgs &a, int num_sms, cudaStream_t stream) {
    if (a.pairs < 1) return cudaSuccess;
    const size_t smem = sizeof(uint32_t) * 5 * (size_t)((a.nK + 31) / 32);
    int64_t grid = a.pairs;
    if (grid > (int64_t)num_sms * 16) grid = (int64_t)num_sms * 16;
    pair_union_kernel<<<(unsigned)grid, kUnionThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_attention(const AttnArgs &a, const AttnMaps &maps, int num_sms,
                             cudaStream_t stream) {
    if (a.pairs < 1) return cudaSuccess;
    return a.D == 128 ? launch_attn_d<128>(a, maps, num_sms, stream)
                      : launch_attn_d<64>(a, maps, num_sms, stream);
}

}  // namespace abatt
