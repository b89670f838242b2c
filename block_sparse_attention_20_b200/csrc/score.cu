// score.cu -- IBCS part 2: every centroid's softmax mass per key block, and
// the per-query-block combination into block probabilities p ("Accurate
// Block Attention", abstract, selector sentence: the clustered queries
// estimate block importance).
//
// keys_f16_kernel: the keys once to fp16, the scoring GEMM's B operand.
//
// score_mass_kernel: one CTA per (head, 128 centroid rows, key-range chunk).
// The centroid tile (fp16 of the pre-scaled fp32 centroids: 11 significant
// bits, against 8 for bf16) stays in shared memory; 128-key fp16 tiles of K
// stream through a 4-stage TMA ring; one warp issues tcgen05 MMAs
// (kind::f16, fp32 accumulation) into four 128x128 accumulator buffers
// in tensor memory; four epilogue warpgroups (one per accumulator buffer,
// thread = centroid row) turn each tile into base-2 exponentials relative to
// the row's running maximum and sum them per key block, two values per
// packed fp32 instruction, with a fixed share of the exponentials on the FMA
// pipe (polynomial) and the rest on the special-function unit.  The partial
// block sums of a tile are written with the reference maximum they were
// taken against, so no second pass over the keys is needed.
//
// combine_kernel: one CTA per query block:
//   p_b = sum_j (n_j/n) * r_{j,b} * 2^(mref_{j,T(b)} - m_j) / Z_j
// where (m_j, Z_j) is centroid j's final running maximum and sum.
#include "kernels.cuh"

namespace abatt {

namespace {

constexpr int kScoreStages = 4;
constexpr int kScoreEpi = 4;        // epilogue warpgroups = accumulator buffers in tensor memory
constexpr int kScoreThreads = kScoreEpi * 128 + 64;  // + a TMA warp and an MMA warp
constexpr int kWarpTma = kScoreEpi * 4, kWarpMma = kScoreEpi * 4 + 1;
#define kNegInf (-__int_as_float(0x7f800000))
// exponent pairs of every sixteen that the epilogue evaluates with the
// FMA-pipe polynomial (the others use ex2)
#ifndef ABATT_SCORE_POLY_OF_16
#define ABATT_SCORE_POLY_OF_16 4
#endif
constexpr int kScorePolyOf16 = ABATT_SCORE_POLY_OF_16;

__device__ __forceinline__ uint32_t bf16x2_to_f16x2_sat(uint32_t w) {
    const float lo = fminf(fmaxf(__uint_as_float(w << 16), -65504.0f), 65504.0f);
    const float hi = fminf(fmaxf(__uint_as_float(w & 0xffff0000u), -65504.0f), 65504.0f);
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__global__ void __launch_bounds__(256) keys_f16_kernel(const uint4 *__restrict__ src,
                                                       uint4 *__restrict__ dst, int64_t n8) {
    const int64_t stride = (int64_t)gridDim.x * 256;
    for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n8; i += 2 * stride) {
        const bool two = i + stride < n8;
        const uint4 u0 = __ldg(src + i);
        const uint4 u1 = two ? __ldg(src + i + stride) : make_uint4(0, 0, 0, 0);
        dst[i] = make_uint4(bf16x2_to_f16x2_sat(u0.x), bf16x2_to_f16x2_sat(u0.y),
                            bf16x2_to_f16x2_sat(u0.z), bf16x2_to_f16x2_sat(u0.w));
        if (two)
            dst[i + stride] = make_uint4(bf16x2_to_f16x2_sat(u1.x), bf16x2_to_f16x2_sat(u1.y),
                                         bf16x2_to_f16x2_sat(u1.z), bf16x2_to_f16x2_sat(u1.w));
    }
}

// strided keys: thread = (row bh*N + t, 8 dims)
__global__ void __launch_bounds__(256) keys_f16_strided_kernel(const __nv_bfloat16 *__restrict__ K,
                                                               const Strides st, uint4 *__restrict__ dst,
                                                               int64_t heads, int N, int D) {
    const int cpr = D / 8;
    const int64_t total = heads * (int64_t)N * cpr;
    for (int64_t w = (int64_t)blockIdx.x * 256 + threadIdx.x; w < total; w += (int64_t)gridDim.x * 256) {
        const int x8 = (int)(w % cpr);
        const int64_t row = w / cpr;
        const int t = (int)(row % N);
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(K + st.head_base(row / N) + t * st.sT) + x8);
        dst[w] = make_uint4(bf16x2_to_f16x2_sat(u.x), bf16x2_to_f16x2_sat(u.y), bf16x2_to_f16x2_sat(u.z),
                            bf16x2_to_f16x2_sat(u.w));
    }
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int BPT>
__device__ __forceinline__ void store_blocks(float *dst, const float (&bs)[BPT]) {
    if constexpr (BPT % 4 == 0) {
#pragma unroll
        for (int k = 0; k < BPT; k += 4)
            *reinterpret_cast<float4 *>(dst + k) = make_float4(bs[k], bs[k + 1], bs[k + 2], bs[k + 3]);
    } else if constexpr (BPT == 2) {
        *reinterpret_cast<float2 *>(dst) = make_float2(bs[0], bs[1]);
    } else {
        dst[0] = bs[0];
    }
}

template <int D, int BK>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_mass_kernel(const __grid_constant__ ScoreMaps maps, const ScoreArgs a) {
    constexpr int CH = D / 64;
    constexpr uint32_t TILE = 128u * D * 2u;
    constexpr int BPT = 128 / BK;
    constexpr int ST = kScoreStages;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sA = smem;
    uint8_t *sK = smem + TILE;

    __shared__ __align__(8) uint64_t bar_a;
    __shared__ __align__(8) uint64_t bar_kfull[ST], bar_kempty[ST];
    __shared__ __align__(8) uint64_t bar_sfull[kScoreEpi], bar_sempty[kScoreEpi];
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    __shared__ float2 mz_s[kScoreEpi][128];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = blockIdx.x, hd = blockIdx.y, chunk = blockIdx.z;
    // this CTA's key tiles: [kt0, kt0 + ntl)
    const int kt0 = chunk * a.chunk_tiles;
    const int ntl = min(a.chunk_tiles, a.nT - kt0);
    __shared__ int skip_s;
    // a bounded wait elsewhere already gave up: do not start more work.  One
    // read, shared by the whole CTA, so every role takes the same decision
    if (threadIdx.x == 0)
        skip_s = a.hdr && (*reinterpret_cast<volatile uint32_t *>(&a.hdr->status) & ABATT_DEVFLAG_TIMEOUT);
    __syncthreads();
    if (skip_s) return;
    const WaitCtx wc{&abort_s, a.hdr, a.wait_ns};

    if (threadIdx.x == 0) {
        abort_s = 0;
        mbar_init(&bar_a, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(&bar_kfull[s], 1);
            mbar_init(&bar_kempty[s], 1);
        }
        for (int b = 0; b < kScoreEpi; ++b) {
            mbar_init(&bar_sfull[b], 1);
            mbar_init(&bar_sempty[b], 4);
        }
        fence_barrier_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(&tmem_base_s, 128 * kScoreEpi);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;

    int issued = 0;       // TMA role: K tiles issued
    int committed = -1;   // MMA role: last K tile whose MMAs were committed

    if (warp == kWarpTma) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&maps.a);
            tma_prefetch_desc(&maps.k);
            mbar_arrive_expect_tx(&bar_a, TILE);
            for (int c = 0; c < CH; ++c) tma_load_3d(sA + c * 16384, &maps.a, &bar_a, c * 64, mt * 128, hd);
            for (int i = 0; i < ntl; ++i) {
                const int s = i % ST;
                if (a.stall && i >= 1) break;  // test hook: no copy after the CTA's first key tile
                if (i >= ST && !mbar_wait(&bar_kempty[s], ((i / ST) - 1) & 1, wc, 0x101)) break;
                mbar_arrive_expect_tx(&bar_kfull[s], TILE);
                for (int c = 0; c < CH; ++c)
                    tma_load_3d(sK + s * TILE + c * 16384, &maps.k, &bar_kfull[s], c * 64, (kt0 + i) * 128, hd);
                issued = i + 1;
            }
        }
    } else if (warp == kWarpMma) {
        // ------------------------------ MMA issuer --------------------------------
        // the whole warp follows the schedule (warp-uniform control flow and
        // descriptors); one elected lane issues each tcgen05 instruction
        auto wait_all = [&](uint64_t *bar, uint32_t parity, uint32_t site) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc, site));
        };
        if (wait_all(&bar_a, 0, 0x102)) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_f16(128, 128);
            const uint64_t da = sdesc_sw128(smem_u32(sA), 16, 1024);
            const bool fill = BK != 1 || a.mode != 2;  // the epilogue leaves -m_ref in the buffer
            for (int i = 0; i < ntl; ++i) {
                const int s = i % ST, buf = i % kScoreEpi, use = i / kScoreEpi;
                if (!wait_all(&bar_kfull[s], (i / ST) & 1, 0x103)) break;
                if (use > 0 && !wait_all(&bar_sempty[buf], (use - 1) & 1, 0x104)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + buf * 128;
                const uint64_t kd = sdesc_sw128(smem_u32(sK + s * TILE), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
                    // after a buffer's first tile the epilogue leaves -m_ref in it:
                    // accumulate onto it, so the product arrives as x - m_ref
                    umma_ss_w(d_tmem, da + off, kd + off, idesc, (kk > 0 || (use > 0 && fill)) ? 1u : 0u);
                }
                umma_commit_w(&bar_kempty[s]);
                umma_commit_w(&bar_sfull[buf]);
                committed = i;
            }
        }
    } else {
        // ------------------------------ epilogue ----------------------------------
        // Warpgroup e takes the tiles i = e (mod kScoreEpi) from accumulator
        // buffer e, 32 columns at a time in two passes (the tile maximum, then
        // the exponentials), so a thread holds 32 scores, not 128.
        const int e = warp >> 2;        // accumulator buffer of this warpgroup
        const int wq = warp & 3;        // TMEM lane quarter
        const int rl = wq * 32 + lane;  // centroid row within the tile
        const int grow = mt * 128 + rl;
        const bool valid = grow < a.MC;
        const int64_t gr = (int64_t)hd * a.MC + grow;
        float m_run = kNegInf, Z = 0.0f;  // reference (base 2) and sum relative to it
        // coarse mode 2: this row's final maximum m_j and log2(w_j / Z_j)
        float mj = 0.0f, lfj = kNegInf;
        if (BK == 1 && a.mode == 2 && valid) {
            const float2 *q = a.mz + gr * a.nchunk;
            float m = kNegInf;
            for (int c = 0; c < a.nchunk; ++c) m = fmaxf(m, q[c].x);
            float z = 0.0f;
            for (int c = 0; c < a.nchunk; ++c)
                if (q[c].x != kNegInf) z += q[c].y * ex2_approx(q[c].x - m);
            const float w = a.weight[gr];
            if (w > 0.0f && z > 0.0f) {
                mj = m;
                lfj = __log2f(w / z);
            }
        }
        for (int i = e; i < ntl; i += kScoreEpi) {
            const int kt = kt0 + i, use = i / kScoreEpi;
            // warp-uniform outcome: the lanes go on to warp-collective tcgen05 loads
            if (!__all_sync(0xffffffffu, mbar_wait(&bar_sfull[e], use & 1, wc, 0x105))) break;
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(wq * 32) << 16) + e * 128;
            const int nvalid = min(128, a.N - kt * 128);  // < 128 only on the sequence's last tile
            auto load = [&](int q, uint32_t (&v)[32]) {
                tmem_ld32(taddr + q * 32, v);
                tmem_wait_ld();
                if (nvalid < 128) {  // keys past N count for nothing
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (q * 32 + c >= nvalid) v[c] = __float_as_uint(kNegInf);
                }
            };
            bool emitted = false;
            if constexpr (BK == 1) {
              if (a.mode == 2) {
                emitted = true;
                // coarse scoring, second pass: e_{j,b} = (w_j/Z_j) 2^(x_jb - m_j), summed
                // over the C centroid rows of each query block -- C adjacent lanes --
                // by a butterfly reduce-scatter, after which lane g of a group holds
                // the sums of W = 32/C consecutive columns and stores them to p
                const int qi = grow / a.C;
                float *prow = a.p + ((int64_t)hd * (a.MC / a.C) + qi) * a.N;
                const int W = 32 / a.C;
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    uint32_t v[32];
                    load(q, v);
                    const int col0 = kt * 128 + q * 32;
                    float x[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) x[c] = ex2_approx((__uint_as_float(v[c]) - mj) + lfj);
                    const int lastc = a.N - 1 - col0;  // the last block, weighted by n_last / Bk
                    if (lastc >= 0 && lastc < 32) {
#pragma unroll
                        for (int c = 0; c < 32; ++c)
                            if (c == lastc) x[c] *= a.last_weight;
                    }
                    int s = a.C >> 1;
#pragma unroll
                    for (int k = 0; k < 5; ++k) {
                        const int half = 16 >> k;  // values exchanged at this step
                        if (s > 0) {
                            const bool hi = (lane & s) != 0;
#pragma unroll
                            for (int u = 0; u < half; ++u) {
                                const float send = hi ? x[u] : x[u + half];
                                const float keep = hi ? x[u + half] : x[u];
                                x[u] = keep + __shfl_xor_sync(0xffffffffu, send, s);
                            }
                            s >>= 1;
                        }
                    }
                    const int cb = col0 + (lane & (a.C - 1)) * W;
                    if (valid) {
#pragma unroll
                        for (int k = 0; k < 32; ++k)
                            if (k < W && cb + k < a.N) prow[cb + k] = x[k];
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_sempty[e]);
              }
            }
            if (emitted) {
            } else if constexpr (BK == 1) {
                // coarse scoring: every column of the tile is one key block (its
                // mean key); each tile takes the exact path and stores one value per
                // column, the last block weighted by its share of a full block
                float tq[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t v[32];
                    load(q, v);
                    float t0 = kNegInf, t1 = kNegInf;
#pragma unroll
                    for (int c = 0; c < 32; c += 4) {
                        t0 = fmax3f(t0, __uint_as_float(v[c]), __uint_as_float(v[c + 1]));
                        t1 = fmax3f(t1, __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
                    }
                    tq[q] = fmaxf(t0, t1);
                }
                const float mx = fmaxf(fmax3f(tq[0], tq[1], tq[2]), tq[3]);
                const float base = (m_run == kNegInf) ? 0.0f : m_run;  // what y is relative to
                const float m_new = fmaxf(m_run, base + mx);
                const float alpha = (m_run == kNegInf) ? 0.0f : ex2_approx(m_run - m_new);
                Z *= alpha;
                m_run = m_new;
                const float sub = m_new - base;
                float zt = 0.0f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t v[32];
                    load(q, v);
                    float4 *dst = reinterpret_cast<float4 *>(a.r + gr * a.ldr + (int64_t)kt * 128 + q * 32);
                    const int col0 = kt * 128 + q * 32;  // key column of v[0]
#pragma unroll
                    for (int c = 0; c < 32; c += 4) {
                        float4 e4 = make_float4(ex2_approx(__uint_as_float(v[c]) - sub),
                                                ex2_approx(__uint_as_float(v[c + 1]) - sub),
                                                ex2_approx(__uint_as_float(v[c + 2]) - sub),
                                                ex2_approx(__uint_as_float(v[c + 3]) - sub));
                        const int last = a.N - 1 - (col0 + c);  // 0..3: the last block is here
                        if (last >= 0 && last < 4) {
                            if (last == 0) e4.x *= a.last_weight;
                            else if (last == 1) e4.y *= a.last_weight;
                            else if (last == 2) e4.z *= a.last_weight;
                            else e4.w *= a.last_weight;
                        }
                        zt += (e4.x + e4.y) + (e4.z + e4.w);
                        if (valid && a.mode == 0) dst[c / 4] = e4;
                    }
                }
                Z += zt;
                if (i + kScoreEpi < ntl) {
                    const uint32_t nmr = __float_as_uint(m_run == kNegInf ? 0.0f : -m_run);
#pragma unroll
                    for (int q = 0; q < 4; ++q) tmem_fill32(taddr + q * 32, nmr);
                    tmem_wait_st();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_sempty[e]);
                if (valid && a.mode == 0) a.mref[gr * a.nT + kt] = m_run;
            } else {
                // block sums of 2^(y - sub) over the tile, y the buffer's values
                constexpr int NA = BPT >= 8 ? 1 : 8 / BPT;
                float bs[BPT];
                auto block_sums = [&](float sub) {
                    const float2 nm = make_float2(-sub, -sub);
                    float2 acc[BPT][NA];
#pragma unroll
                    for (int k = 0; k < BPT; ++k)
#pragma unroll
                        for (int u = 0; u < NA; ++u) acc[k][u] = make_float2(0.0f, 0.0f);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t v[32];
                        load(q, v);
#pragma unroll
                        for (int c = 0; c < 32; c += 2) {
                            const int col = q * 32 + c;
                            float2 x = make_float2(__uint_as_float(v[c]), __uint_as_float(v[c + 1]));
                            if (sub != 0.0f) x = __fadd2_rn(x, nm);
                            float2 ex;
                            if (((col >> 1) & 15) < kScorePolyOf16) {
                                // the polynomial is valid below 2^128: larger inputs land at
                                // 2^100 and send the tile to the exact path below
                                x.x = fminf(x.x, 100.0f);
                                x.y = fminf(x.y, 100.0f);
                                ex = exp2_poly2<4>(x);
                            } else {
                                ex.x = ex2_approx(x.x);
                                ex.y = ex2_approx(x.y);
                            }
                            float2 &s2 = acc[col / BK][(col >> 1) % NA];
                            s2 = __fadd2_rn(s2, ex);
                        }
                    }
#pragma unroll
                    for (int k = 0; k < BPT; ++k) {
                        float2 t2 = acc[k][0];
#pragma unroll
                        for (int u = 1; u < NA; ++u) t2 = __fadd2_rn(t2, acc[k][u]);
                        bs[k] = t2.x + t2.y;
                    }
                };
                // exact path: the tile's own maximum mx of y (relative to the current
                // reference, or absolute on the first tile) becomes part of the reference
                auto exact = [&]() {
                    float tq[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t v[32];
                        load(q, v);
                        float t0 = kNegInf, t1 = kNegInf;
#pragma unroll
                        for (int c = 0; c < 32; c += 4) {
                            t0 = fmax3f(t0, __uint_as_float(v[c]), __uint_as_float(v[c + 1]));
                            t1 = fmax3f(t1, __uint_as_float(v[c + 2]), __uint_as_float(v[c + 3]));
                        }
                        tq[q] = fmaxf(t0, t1);
                    }
                    const float mx = fmaxf(fmax3f(tq[0], tq[1], tq[2]), tq[3]);
                    const float base = (m_run == kNegInf) ? 0.0f : m_run;  // what y is relative to
                    const float m_new = fmaxf(m_run, base + mx);
                    const float alpha = (m_run == kNegInf) ? 0.0f : ex2_approx(m_run - m_new);
                    Z *= alpha;
                    m_run = m_new;
                    block_sums(m_new - base);
                };
                // first tile of this buffer (the MMA started from zero): exact path;
                // later tiles: the buffer held -m_run, so y = x - m_run already, one
                // pass of exponentials -- unless some row's scores outgrew its
                // reference, then the warp redoes the tile with the exact maximum
                // (correct for every row; tensor-memory loads stay warp-uniform)
                bool redo = use == 0;
                if (!redo) {
                    block_sums(0.0f);
                    float big = 0.0f;
#pragma unroll
                    for (int k = 0; k < BPT; ++k) big = fmaxf(big, bs[k]);
                    redo = __any_sync(0xffffffffu, !(big < 0x1p80f));
                }
                if (redo) exact();
                // leave -m_run in the buffer for its next tile, then free it
                if (i + kScoreEpi < ntl) {
                    const uint32_t nmr = __float_as_uint(m_run == kNegInf ? 0.0f : -m_run);
#pragma unroll
                    for (int q = 0; q < 4; ++q) tmem_fill32(taddr + q * 32, nmr);
                    tmem_wait_st();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_sempty[e]);
#pragma unroll
                for (int k = 0; k < BPT; ++k) Z += bs[k];
                if (valid) {
                    store_blocks<BPT>(a.r + gr * a.ldr + (int64_t)kt * BPT, bs);
                    a.mref[gr * a.nT + kt] = m_run;
                }
            }
        }
        mz_s[e][rl] = make_float2(m_run, Z);
        tc_fence_before();
        __syncthreads();
        if (e == 0) {
            // merge the warpgroups' (max, sum) of this row
            float m = kNegInf;
#pragma unroll
            for (int g = 0; g < kScoreEpi; ++g) m = fmaxf(m, mz_s[g][rl].x);
            float z = 0.0f;
#pragma unroll
            for (int g = 0; g < kScoreEpi; ++g) {
                const float2 o = mz_s[g][rl];
                if (o.x != kNegInf) z += o.y * ex2_approx(o.x - m);
            }
            if (valid && (BK != 1 || a.mode != 2)) a.mz[gr * a.nchunk + chunk] = make_float2(m, z);
        }
    }
    if (warp >= kWarpTma) {
        tc_fence_before();
        __syncthreads();  // pairs with the epilogue's barrier above
    }

    // ------------------------------ teardown --------------------------------------
    if (abort_s) {
        // drain copies and MMAs still in flight before shared/tensor memory go away
        if (warp == kWarpTma && lane == 0)
            for (int t = issued - ST > 0 ? issued - ST : 0; t < issued; ++t) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&bar_kfull[t % ST], (t / ST) & 1) &&
                       globaltimer_ns() - t0 < a.wait_ns) {
                }
            }
        if (warp == kWarpMma && lane == 0 && committed >= 0) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&bar_kempty[committed % ST], (committed / ST) & 1) &&
                   globaltimer_ns() - t0 < a.wait_ns) {
            }
        }
    }
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 128 * kScoreEpi);
    }
}

template <int BPT>
__global__ void __launch_bounds__(256) combine_kernel(const CombineArgs a) {
    __shared__ float f_s[16], m_s[16];
    for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
        __syncthreads();
        if (threadIdx.x < a.C) {
            const int64_t j = row * a.C + threadIdx.x;
            const float w = a.weight[j];
            // the key range was split into chunks: merge their (max, sum)
            const float2 *mzj = a.mz + j * a.nchunk;
            float m = kNegInf;
            for (int c = 0; c < a.nchunk; ++c) m = fmaxf(m, mzj[c].x);
            float z = 0.0f;
            for (int c = 0; c < a.nchunk; ++c) {
                const float2 q = mzj[c];
                if (q.x != kNegInf) z += q.y * ex2_approx(q.x - m);
            }
            f_s[threadIdx.x] = (w > 0.0f && z > 0.0f) ? w / z : 0.0f;
            m_s[threadIdx.x] = m;
        }
        __syncthreads();
        float *prow = a.p + row * (int64_t)a.nK;
        for (int T = threadIdx.x; T < a.nT; T += blockDim.x) {
            float acc[BPT];
#pragma unroll
            for (int k = 0; k < BPT; ++k) acc[k] = 0.0f;
            // four centroids at a time: all their loads in flight before use
            for (int j0 = 0; j0 < a.C; j0 += 4) {
                float mr[4], rv[4][BPT];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = j0 + u;
                    mr[u] = 0.0f;
#pragma unroll
                    for (int k = 0; k < BPT; ++k) rv[u][k] = 0.0f;
                    if (j < a.C) {
                        const int64_t cj = row * a.C + j;
                        mr[u] = __ldg(a.mref + cj * a.nT + T);
                        const float *rr = a.r + cj * a.ldr + (int64_t)T * BPT;
                        if constexpr (BPT % 4 == 0) {
#pragma unroll
                            for (int k = 0; k < BPT; k += 4) {
                                const float4 q = __ldg(reinterpret_cast<const float4 *>(rr + k));
                                rv[u][k] = q.x; rv[u][k + 1] = q.y; rv[u][k + 2] = q.z; rv[u][k + 3] = q.w;
                            }
                        } else {
#pragma unroll
                            for (int k = 0; k < BPT; ++k) rv[u][k] = __ldg(rr + k);
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = j0 + u;
                    if (j >= a.C) break;
                    const float f = f_s[j];
                    if (f == 0.0f) continue;
                    const float coef = f * ex2_approx(mr[u] - m_s[j]);
#pragma unroll
                    for (int k = 0; k < BPT; ++k) acc[k] = fmaf(coef, rv[u][k], acc[k]);
                }
            }
#pragma unroll
            for (int k = 0; k < BPT; ++k) {
                const int b = T * BPT + k;
                if (b < a.nK) prow[b] = acc[k];
            }
        }
    }
}

// ---- coarse scoring ------------------------------------------------------------
// Kbar[h][b][x] = fp16 of the mean of K[h][b*Bk .. b*Bk + n_b)[x]; thread = (h, b, 8 dims)
__global__ void __launch_bounds__(256) keys_block_mean_kernel(const __nv_bfloat16 *__restrict__ K,
                                                              const Strides st, __half *__restrict__ Kbar,
                                                              int64_t heads, int N, int D, int Bk, int nK) {
    const int cpr = D / 8;  // 8-dim chunks per key
    const int64_t total = heads * (int64_t)nK * cpr;
    for (int64_t w = (int64_t)blockIdx.x * 256 + threadIdx.x; w < total; w += (int64_t)gridDim.x * 256) {
        const int x8 = (int)(w % cpr);
        const int64_t hb = w / cpr;
        const int b = (int)(hb % nK);
        const int64_t h = hb / nK;
        const int n = min(Bk, N - b * Bk);
        const __nv_bfloat16 *src = K + st.head_base(h) + (int64_t)b * Bk * st.sT + x8 * 8;
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int u = 0; u < n; ++u) {
            const uint4 q = __ldg(reinterpret_cast<const uint4 *>(src + (int64_t)u * st.sT));
            const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                acc[2 * k] += __uint_as_float(wv[k] << 16);
                acc[2 * k + 1] += __uint_as_float(wv[k] & 0xffff0000u);
            }
        }
        const float inv = 1.0f / (float)n;
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float lo = fminf(fmaxf(acc[2 * k] * inv, -65504.0f), 65504.0f);
            const float hi = fminf(fmaxf(acc[2 * k + 1] * inv, -65504.0f), 65504.0f);
            const __half2 h2 = __floats2half2_rn(lo, hi);
            o[k] = *reinterpret_cast<const uint32_t *>(&h2);
        }
        reinterpret_cast<uint4 *>(Kbar + hb * D)[x8] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// p_b = sum_j (n_j/n) * r_{j,b} * 2^(mref_{j,b/128} - m_j) / Z_j, one thread per block
__global__ void __launch_bounds__(256) combine_cols_kernel(const CombineArgs a) {
    extern __shared__ float coef_s[];  // [C][nT]: (n_j/n) / Z_j * 2^(mref - m_j)
    __shared__ float f_s[16], m_s[16];
    for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
        __syncthreads();
        if (threadIdx.x < a.C) {
            const int64_t j = row * a.C + threadIdx.x;
            const float w = a.weight[j];
            const float2 *mzj = a.mz + j * a.nchunk;
            float m = kNegInf;
            for (int c = 0; c < a.nchunk; ++c) m = fmaxf(m, mzj[c].x);
            float z = 0.0f;
            for (int c = 0; c < a.nchunk; ++c) {
                const float2 q = mzj[c];
                if (q.x != kNegInf) z += q.y * ex2_approx(q.x - m);
            }
            f_s[threadIdx.x] = (w > 0.0f && z > 0.0f) ? w / z : 0.0f;
            m_s[threadIdx.x] = m;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < a.C * a.nT; e += blockDim.x) {
            const int j = e / a.nT, T = e % a.nT;
            const float f = f_s[j];
            coef_s[e] = f == 0.0f ? 0.0f : f * ex2_approx(__ldg(a.mref + (row * a.C + j) * a.nT + T) - m_s[j]);
        }
        __syncthreads();
        float *prow = a.p + row * (int64_t)a.nK;
        // four blocks per thread (one float4 of r; rows of r are padded to 128
        // columns, zeros past nK), the loads of four centroids in flight at once
        for (int b = threadIdx.x * 4; b < a.nK; b += blockDim.x * 4) {
            const int T = b >> 7;
            float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            for (int j0 = 0; j0 < a.C; j0 += 4) {
                float4 rv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    rv[u] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    if (j0 + u < a.C)
                        rv[u] = __ldg(reinterpret_cast<const float4 *>(a.r + (row * a.C + j0 + u) * a.ldr + b));
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (j0 + u >= a.C) break;
                    const float c = coef_s[(j0 + u) * a.nT + T];
                    acc.x = fmaf(c, rv[u].x, acc.x);
                    acc.y = fmaf(c, rv[u].y, acc.y);
                    acc.z = fmaf(c, rv[u].z, acc.z);
                    acc.w = fmaf(c, rv[u].w, acc.w);
                }
            }
            if (b + 3 < a.nK && (a.nK & 3) == 0) {
                *reinterpret_cast<float4 *>(prow + b) = acc;
            } else {
                const float v[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (b + k < a.nK) prow[b + k] = v[k];
            }
        }
    }
}

template <int D, int BK>
cudaError_t launch_score_t(const ScoreArgs &a, const ScoreMaps &maps, cudaStream_t stream) {
    const size_t smem = (1 + kScoreStages) * (size_t)(128 * D * 2) + 1024;
    cudaError_t e = cudaFuncSetAttribute(score_mass_kernel<D, BK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.MC + 127) / 128, a.heads, a.nchunk);
    score_mass_kernel<D, BK><<<grid, kScoreThreads, smem, stream>>>(maps, a);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_score_d(const ScoreArgs &a, const ScoreMaps &maps, cudaStream_t stream) {
    switch (a.Bk) {
        case 1: return launch_score_t<D, 1>(a, maps, stream);  // coarse: one column per key block
        case 16: return launch_score_t<D, 16>(a, maps, stream);
        case 32: return launch_score_t<D, 32>(a, maps, stream);
        case 64: return launch_score_t<D, 64>(a, maps, stream);
        case 128: return launch_score_t<D, 128>(a, maps, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_score(const ScoreArgs &a, const ScoreMaps &maps, int, cudaStream_t stream) {
    if (a.heads < 1 || a.MC < 1 || a.nT < 1) return cudaSuccess;
    return a.D == 128 ? launch_score_d<128>(a, maps, stream) : launch_score_d<64>(a, maps, stream);
}

cudaError_t launch_keys_f16(const __nv_bfloat16 *K, __half *K16, int64_t n8, int num_sms,
                            cudaStream_t stream) {
    if (n8 < 1) return cudaSuccess;
    int64_t grid = (n8 + 511) / 512;
    const int64_t cap = (int64_t)num_sms * 8;
    if (grid > cap) grid = cap;
    keys_f16_kernel<<<(unsigned)grid, 256, 0, stream>>>(reinterpret_cast<const uint4 *>(K),
                                                        reinterpret_cast<uint4 *>(K16), n8);
    return cudaGetLastError();
}

cudaError_t launch_keys_f16_strided(const __nv_bfloat16 *K, const Strides &st, __half *K16, int64_t heads,
                                    int N, int D, int num_sms, cudaStream_t stream) {
    const int64_t total = heads * (int64_t)N * (D / 8);
    if (total < 1) return cudaSuccess;
    int64_t grid = (total + 255) / 256;
    const int64_t cap = (int64_t)num_sms * 8;
    if (grid > cap) grid = cap;
    keys_f16_strided_kernel<<<(unsigned)grid, 256, 0, stream>>>(K, st, reinterpret_cast<uint4 *>(K16), heads,
                                                                N, D);
    return cudaGetLastError();
}

cudaError_t launch_keys_block_mean(const __nv_bfloat16 *K, const Strides &st, __half *Kbar, int64_t heads,
                                   int N, int D, int Bk, int nK, int num_sms, cudaStream_t stream) {
    const int64_t total = heads * (int64_t)nK * (D / 8);
    if (total < 1) return cudaSuccess;
    int64_t grid = (total + 255) / 256;
    const int64_t cap = (int64_t)num_sms * 8;
    if (grid > cap) grid = cap;
    keys_block_mean_kernel<<<(unsigned)grid, 256, 0, stream>>>(K, st, Kbar, heads, N, D, Bk, nK);
    return cudaGetLastError();
}

cudaError_t launch_combine_cols(const CombineArgs &a, int num_sms, cudaStream_t stream) {
    int64_t grid = a.rows;
    const int64_t cap = (int64_t)num_sms * 16;
    if (grid > cap) grid = cap;
    if (grid < 1) return cudaSuccess;
    const size_t smem = sizeof(float) * (size_t)a.C * a.nT;
    combine_cols_kernel<<<(unsigned)grid, 256, smem, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_combine(const CombineArgs &a, int num_sms, cudaStream_t stream) {
    int64_t grid = a.rows;
    const int64_t cap = (int64_t)num_sms * 16;
    if (grid > cap) grid = cap;
    if (grid < 1) return cudaSuccess;
    switch (128 / a.Bk) {
        case 8: combine_kernel<8><<<(unsigned)grid, 256, 0, stream>>>(a); break;
        case 4: combine_kernel<4><<<(unsigned)grid, 256, 0, stream>>>(a); break;
        case 2: combine_kernel<2><<<(unsigned)grid, 256, 0, stream>>>(a); break;
        default: combine_kernel<1><<<(unsigned)grid, 256, 0, stream>>>(a); break;
    }
    return cudaGetLastError();
}

}  // namespace abatt
