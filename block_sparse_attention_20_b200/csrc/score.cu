// score.cu -- IBCS part 2: every centroid's softmax mass per key block, and
// the per-query-block combination into block probabilities p ("Accurate
// Block Attention", abstract, selector sentence: the clustered queries
// estimate block importance).
//
// score_mass_kernel: one CTA per (head, 128 centroid rows).  The centroid
// tile (bf16 hi + lo split of the pre-scaled fp32 centroids) stays in shared
// memory; 128-key tiles of K stream through a 4-stage TMA ring; one thread
// issues tcgen05 MMAs into a double-buffered 128x128 fp32 accumulator in
// tensor memory; two epilogue warpgroups (one per accumulator buffer, thread
// = centroid row) turn each tile into base-2 exponentials relative to the
// row's running maximum and sum them per key block.  The partial block sums
// of a tile are written with the reference maximum they were taken against,
// so no second pass over the keys is needed.
//
// combine_kernel: one CTA per query block:
//   p_b = sum_j (n_j/n) * r_{j,b} * 2^(mref_{j,T(b)} - m_j) / Z_j
// where (m_j, Z_j) is centroid j's final running maximum and sum.
#include "kernels.cuh"

namespace abatt {

namespace {

constexpr int kScoreStages = 4;
constexpr int kScoreThreads = 320;  // warps 0-7 epilogue (2 warpgroups), 8 TMA, 9 MMA
#define kNegInf (-__int_as_float(0x7f800000))

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
    uint8_t *sA_hi = smem;
    uint8_t *sA_lo = smem + TILE;
    uint8_t *sK = smem + 2 * TILE;

    __shared__ __align__(8) uint64_t bar_a;
    __shared__ __align__(8) uint64_t bar_kfull[ST], bar_kempty[ST];
    __shared__ __align__(8) uint64_t bar_sfull[2], bar_sempty[2];
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    __shared__ float2 mz_s[128];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = blockIdx.x, hd = blockIdx.y, chunk = blockIdx.z;
    // this CTA's key tiles: [kt0, kt0 + ntl)
    const int kt0 = chunk * a.chunk_tiles;
    const int ntl = min(a.chunk_tiles, a.nT - kt0);
    // a bounded wait elsewhere already gave up: do not start more work
    if (a.hdr && (*reinterpret_cast<volatile uint32_t *>(&a.hdr->status) & ABATT_DEVFLAG_TIMEOUT))
        return;
    const WaitCtx wc{&abort_s, a.hdr, a.wait_ns};

    if (threadIdx.x == 0) {
        abort_s = 0;
        mbar_init(&bar_a, 1);
        for (int s = 0; s < ST; ++s) {
            mbar_init(&bar_kfull[s], 1);
            mbar_init(&bar_kempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar_sfull[b], 1);
            mbar_init(&bar_sempty[b], 4);
        }
        fence_barrier_init();
    }
    if (warp == 9) {
        tmem_alloc(&tmem_base_s, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;

    int issued = 0;       // TMA role: K tiles issued
    int committed = -1;   // MMA role: last K tile whose MMAs were committed

    if (warp == 8) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&maps.a_hi);
            tma_prefetch_desc(&maps.k);
            mbar_arrive_expect_tx(&bar_a, (a.use_lo ? 2u : 1u) * TILE);
            for (int c = 0; c < CH; ++c) {
                tma_load_3d(sA_hi + c * 16384, &maps.a_hi, &bar_a, c * 64, mt * 128, hd);
                if (a.use_lo) tma_load_3d(sA_lo + c * 16384, &maps.a_lo, &bar_a, c * 64, mt * 128, hd);
            }
            for (int i = 0; i < ntl; ++i) {
                const int s = i % ST;
                if (i >= ST && !mbar_wait(&bar_kempty[s], ((i / ST) - 1) & 1, wc, 0x101)) break;
                mbar_arrive_expect_tx(&bar_kfull[s], TILE);
                for (int c = 0; c < CH; ++c)
                    tma_load_3d(sK + s * TILE + c * 16384, &maps.k, &bar_kfull[s], c * 64, (kt0 + i) * 128, hd);
                issued = i + 1;
            }
        }
    } else if (warp == 9) {
        // ------------------------------ MMA issuer --------------------------------
        // the whole warp follows the schedule (warp-uniform control flow and
        // descriptors); one elected lane issues each tcgen05 instruction
        auto wait_all = [&](uint64_t *bar, uint32_t parity, uint32_t site) -> bool {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc, site));
        };
        if (wait_all(&bar_a, 0, 0x102)) {
            tc_fence_after();
            constexpr uint32_t idesc = idesc_bf16(128, 128);
            const uint32_t a_hi = smem_u32(sA_hi), a_lo = smem_u32(sA_lo);
            const uint64_t dhi = sdesc_sw128(a_hi, 16, 1024), dlo = sdesc_sw128(a_lo, 16, 1024);
            const bool use_lo = a.use_lo != 0;
            for (int i = 0; i < ntl; ++i) {
                const int s = i % ST, buf = i & 1, use = i >> 1;
                if (!wait_all(&bar_kfull[s], (i / ST) & 1, 0x103)) break;
                if (use > 0 && !wait_all(&bar_sempty[buf], (use - 1) & 1, 0x104)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + buf * 128;
                const uint64_t kd = sdesc_sw128(smem_u32(sK + s * TILE), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
                    umma_bf16_ss_w(d_tmem, dhi + off, kd + off, idesc, kk > 0);
                    if (use_lo) umma_bf16_ss_w(d_tmem, dlo + off, kd + off, idesc, 1);
                }
                umma_commit_w(&bar_kempty[s]);
                umma_commit_w(&bar_sfull[buf]);
                committed = i;
            }
        }
    } else {
        // ------------------------------ epilogue ----------------------------------
        const int e = warp >> 2;        // accumulator buffer of this warpgroup
        const int wq = warp & 3;        // TMEM lane quarter
        const int rl = wq * 32 + lane;  // centroid row within the tile
        const int grow = mt * 128 + rl;
        const bool valid = grow < a.MC;
        const int64_t gr = (int64_t)hd * a.MC + grow;
        float m_run = kNegInf, Z = 0.0f;
        for (int i = e; i < ntl; i += 2) {
            const int kt = kt0 + i, use = i >> 1;
            if (!mbar_wait(&bar_sfull[e], use & 1, wc, 0x105)) break;
            tc_fence_after();
            uint32_t v[4][32];
            const uint32_t taddr = tmem + ((uint32_t)(wq * 32) << 16) + e * 128;
            tmem_ld32(taddr + 0, v[0]);
            tmem_ld32(taddr + 32, v[1]);
            tmem_ld32(taddr + 64, v[2]);
            tmem_ld32(taddr + 96, v[3]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_sempty[e]);

            const int kbase = kt * 128;
            const int nvalid = min(128, a.N - kbase);
            if (nvalid < 128) {  // the sequence's last tile: keys past N count for nothing
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (q * 32 + c >= nvalid) v[q][c] = __float_as_uint(kNegInf);
            }
            float tm = kNegInf;
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int c = 0; c < 32; c += 2)
                    tm = fmax3f(tm, __uint_as_float(v[q][c]), __uint_as_float(v[q][c + 1]));
            const float m_new = fmaxf(m_run, tm);
            const float alpha = (m_run == kNegInf) ? 0.0f : ex2_approx(m_run - m_new);
            Z *= alpha;
            m_run = m_new;
            float bs[BPT];
#pragma unroll
            for (int k = 0; k < BPT; ++k) bs[k] = 0.0f;
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    bs[(q * 32 + c) / BK] += ex2_approx(__uint_as_float(v[q][c]) - m_run);
#pragma unroll
            for (int k = 0; k < BPT; ++k) Z += bs[k];
            if (valid) {
                store_blocks<BPT>(a.r + gr * a.ldr + (int64_t)kt * BPT, bs);
                a.mref[gr * a.nT + kt] = m_run;
            }
        }
        if (e == 1) mz_s[rl] = make_float2(m_run, Z);
        tc_fence_before();
        __syncthreads();
        if (e == 0) {
            const float2 o = mz_s[rl];
            const float m = fmaxf(m_run, o.x);
            const float z0 = (m_run == kNegInf) ? 0.0f : Z * ex2_approx(m_run - m);
            const float z1 = (o.x == kNegInf) ? 0.0f : o.y * ex2_approx(o.x - m);
            if (valid) a.mz[gr * a.nchunk + chunk] = make_float2(m, z0 + z1);
        }
    }
    if (warp >= 8) {
        tc_fence_before();
        __syncthreads();  // pairs with the epilogue's barrier above
    }

    // ------------------------------ teardown --------------------------------------
    if (abort_s) {
        // drain copies and MMAs still in flight before shared/tensor memory go away
        if (warp == 8 && lane == 0)
            for (int t = issued - ST > 0 ? issued - ST : 0; t < issued; ++t) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&bar_kfull[t % ST], (t / ST) & 1) &&
                       globaltimer_ns() - t0 < a.wait_ns) {
                }
            }
        if (warp == 9 && lane == 0 && committed >= 0) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&bar_kempty[committed % ST], (committed / ST) & 1) &&
                   globaltimer_ns() - t0 < a.wait_ns) {
            }
        }
    }
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
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

template <int D, int BK>
cudaError_t launch_score_t(const ScoreArgs &a, const ScoreMaps &maps, cudaStream_t stream) {
    const size_t smem = (2 + kScoreStages) * (size_t)(128 * D * 2) + 1024;
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
