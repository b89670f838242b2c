// attention.cu -- gather attention over the drawn key/value blocks
// ("Accurate Block Attention", abstract, kernel sentence: key/value blocks
// much smaller than a tile are gathered into full tensor-core tiles; SIP
// sentence: each drawn block is re-weighted by 1/pi, here as +ln(1/pi) on
// its logits inside the online softmax).
//
// One CTA per query block (128 queries).  Warp roles:
//   warp 0     TMA: Q once; then, per 128-key tile, 128/Bk boxes of Bk rows of
//              K and of V, each landing at its slot of a 128-row 128-byte-
//              swizzled tile (empty slots of the last tile are filled with
//              zeros by loading a box past the end of the tensor);
//   warp 1     tcgen05 MMA issuer: S = Q K^T into a double-buffered 128x128
//              fp32 accumulator in tensor memory, O += P V into a 128xD fp32
//              accumulator in tensor memory;
//   warps 2-5  softmax (thread = query row): base-2 logits plus the block's
//              log-weight, running maximum with a lazy rescale threshold,
//              P in bf16 to shared memory, O correction in tensor memory,
//              final normalisation and bf16 store.
#include "kernels.cuh"

namespace abatt {

namespace {

constexpr int kAttnThreads = 192;
constexpr int kKStages = 2;
constexpr int kVStages = 2;
#define kNegInf (-__int_as_float(0x7f800000))
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // base-2: values up to 2^8 stay in fp32/bf16 range

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int D, int BK>
__global__ void __launch_bounds__(kAttnThreads, 1)
    gather_attn_kernel(const __grid_constant__ AttnMaps maps, const AttnArgs a) {
    constexpr int CH = D / 64;
    constexpr uint32_t TILE = 128u * D * 2u;  // a 128-row operand tile
    constexpr int BPT = 128 / BK;             // blocks per 128-key tile
    constexpr uint32_t TMEM_COLS = 512;       // S0 | S1 | O
    constexpr uint32_t O_COL = 256;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *sQ = smem;
    uint8_t *sK = sQ + TILE;
    uint8_t *sV = sK + kKStages * TILE;
    uint8_t *sP = sV + kVStages * TILE;

    __shared__ __align__(8) uint64_t bar_q, bar_p, bar_pv;
    __shared__ __align__(8) uint64_t bar_kf[kKStages], bar_ke[kKStages];
    __shared__ __align__(8) uint64_t bar_vf[kVStages], bar_ve[kVStages];
    __shared__ __align__(8) uint64_t bar_sf[2], bar_se[2];
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x;
    const int i = (int)(row % a.nQ);
    const int hd = (int)(row / a.nQ);
    const int nrows = min(128, a.N - i * 128);
    const int L = min(max(a.counts[row], 0), a.capacity);
    const int ntiles = (L + BPT - 1) / BPT;
    const int32_t *idx = a.idx + row * (int64_t)a.capacity;
    const float *lw = a.logw + row * (int64_t)a.capacity;
    const int64_t tok0 = (int64_t)hd * a.N + (int64_t)i * 128;

    // a bounded wait elsewhere already gave up: do not start more work
    if (a.hdr && (*reinterpret_cast<volatile uint32_t *>(&a.hdr->status) & ABATT_DEVFLAG_TIMEOUT))
        return;
    if (L == 0) {  // empty list: O = 0, lse = -inf
        for (int e = threadIdx.x; e < nrows * D / 8; e += blockDim.x)
            reinterpret_cast<uint4 *>(a.O + tok0 * D)[e] = make_uint4(0, 0, 0, 0);
        if (a.lse)
            for (int r = threadIdx.x; r < nrows; r += blockDim.x) a.lse[tok0 + r] = kNegInf;
        return;
    }

    const WaitCtx wc{&abort_s, a.hdr, a.wait_ns};
    if (threadIdx.x == 0) {
        abort_s = 0;
        mbar_init(&bar_q, 1);
        mbar_init(&bar_p, 4);
        mbar_init(&bar_pv, 1);
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(&bar_kf[s], 1);
            mbar_init(&bar_ke[s], 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(&bar_vf[s], 1);
            mbar_init(&bar_ve[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar_sf[b], 1);
            mbar_init(&bar_se[b], 4);
        }
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

    int k_issued = 0, v_issued = 0;  // TMA role bookkeeping for the drain
    int committed = 0;               // MMA role: PV tiles committed

    if (warp == 0) {
        // ------------------------------ TMA gather --------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&maps.q);
            tma_prefetch_desc(&maps.k);
            tma_prefetch_desc(&maps.v);
            mbar_arrive_expect_tx(&bar_q, TILE);
            for (int c = 0; c < CH; ++c)
                tma_load_3d(sQ + c * 16384, &maps.q, &bar_q, c * 64, i * 128, hd);
            const int pad_y = a.nK * BK;  // a box starting here lies wholly past N
            bool bad = false;
            for (int t = 0; t <= ntiles; ++t) {
                if (t < ntiles) {
                    const int s = t % kKStages;
                    if (t >= kKStages && !mbar_wait(&bar_ke[s], ((t / kKStages) - 1) & 1, wc, 0x201))
                        break;
                    mbar_arrive_expect_tx(&bar_kf[s], TILE);
                    for (int k = 0; k < BPT; ++k) {
                        const int sidx = t * BPT + k;
                        int y = pad_y;
                        if (sidx < L) {
                            const int b = idx[sidx];
                            if (b >= 0 && b < a.nK) y = b * BK; else bad = true;
                        }
                        for (int c = 0; c < CH; ++c)
                            tma_load_3d(sK + s * TILE + c * 16384 + k * BK * 128, &maps.k, &bar_kf[s],
                                        c * 64, y, hd);
                    }
                    k_issued = t + 1;
                }
                if (t >= 1) {
                    const int tv = t - 1, s = tv % kVStages;
                    if (tv >= kVStages && !mbar_wait(&bar_ve[s], ((tv / kVStages) - 1) & 1, wc, 0x202))
                        break;
                    mbar_arrive_expect_tx(&bar_vf[s], TILE);
                    for (int k = 0; k < BPT; ++k) {
                        const int sidx = tv * BPT + k;
                        int y = pad_y;
                        if (sidx < L) {
                            const int b = idx[sidx];
                            if (b >= 0 && b < a.nK) y = b * BK;
                        }
                        for (int c = 0; c < CH; ++c)
                            tma_load_3d(sV + s * TILE + c * 16384 + k * BK * 128, &maps.v, &bar_vf[s],
                                        c * 64, y, hd);
                    }
                    v_issued = tv + 1;
                }
            }
            if (bad) raise_flag(a.hdr ? &a.hdr->status : nullptr, ABATT_DEVFLAG_BADLIST);
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0 && mbar_wait(&bar_q, 0, wc, 0x203)) {
            constexpr uint32_t idesc_s = idesc_bf16(128, 128);
            constexpr uint32_t idesc_o = idesc_bf16(128, D, /*b_mn_major=*/true);
            const uint32_t q_addr = smem_u32(sQ), p_addr = smem_u32(sP);
            auto issue_s = [&](int t) -> bool {
                const int s = t % kKStages, buf = t & 1;
                if (!mbar_wait(&bar_kf[s], (t / kKStages) & 1, wc, 0x204)) return false;
                if (t >= 2 && !mbar_wait(&bar_se[buf], ((t >> 1) - 1) & 1, wc, 0x205)) return false;
                tc_fence_after();
                const uint32_t k_addr = smem_u32(sK + s * TILE);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    umma_bf16_ss(tmem + buf * 128, sdesc_sw128(q_addr + off, 16, 1024),
                                 sdesc_sw128(k_addr + off, 16, 1024), idesc_s, kk > 0);
                }
                umma_commit(&bar_ke[s]);
                umma_commit(&bar_sf[buf]);
                return true;
            };
            tc_fence_after();
            bool ok = issue_s(0);
            for (int t = 0; ok && t < ntiles; ++t) {
                if (t + 1 < ntiles && !issue_s(t + 1)) break;
                const int s = t % kVStages;
                if (!mbar_wait(&bar_p, t & 1, wc, 0x206)) break;
                if (!mbar_wait(&bar_vf[s], (t / kVStages) & 1, wc, 0x207)) break;
                tc_fence_after();
                const uint32_t v_addr = smem_u32(sV + s * TILE);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t adesc = sdesc_sw128(p_addr + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                    const uint64_t bdesc = sdesc_sw128(v_addr + kk * 2048, 16384, 1024);
                    umma_bf16_ss(tmem + O_COL, adesc, bdesc, idesc_o, (t > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&bar_ve[s]);
                umma_commit(&bar_pv);
                committed = t + 1;
            }
        }
    } else {
        // ------------------------------ softmax -----------------------------------
        const int wq = warp & 3;
        const int r = wq * 32 + lane;  // query row == TMEM lane
        const uint32_t t_lane = (uint32_t)(wq * 32) << 16;
        float m_run = kNegInf, l = 0.0f;
        bool ok = true;
        for (int t = 0; t < ntiles; ++t) {
            // per-slot bias (log-weight in base 2, or -inf) and valid key count
            float bias[BPT];
            int keep[BPT];
#pragma unroll
            for (int k = 0; k < BPT; ++k) {
                const int sidx = t * BPT + k;
                bias[k] = kNegInf;
                keep[k] = 0;
                if (sidx < L) {
                    const int b = idx[sidx];
                    if (b >= 0 && b < a.nK) {
                        bias[k] = lw[sidx] * kLog2e;
                        keep[k] = min(BK, a.N - b * BK);
                    }
                }
            }
            const int buf = t & 1;
            if (!mbar_wait(&bar_sf[buf], (t >> 1) & 1, wc, 0x208)) { ok = false; break; }
            tc_fence_after();
            uint32_t v[4][32];
            const uint32_t sa = tmem + t_lane + buf * 128;
            tmem_ld32(sa + 0, v[0]);
            tmem_ld32(sa + 32, v[1]);
            tmem_ld32(sa + 64, v[2]);
            tmem_ld32(sa + 96, v[3]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_se[buf]);

            float tmax = kNegInf;
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int col = q * 32 + c;
                    float x = fmaf(__uint_as_float(v[q][c]), a.scale_log2, bias[col / BK]);
                    if ((col % BK) >= keep[col / BK]) x = kNegInf;
                    v[q][c] = __float_as_uint(x);
                    tmax = fmaxf(tmax, x);
                }
            const bool need = tmax > m_run + kRescaleThreshold;
            const float m_use = need ? tmax : m_run;
            const float alpha = need ? ((m_run == kNegInf) ? 0.0f : ex2_approx(m_run - tmax)) : 1.0f;
            const float m_sub = (m_use == kNegInf) ? 0.0f : m_use;  // all-masked tile: p = 0
            float rs = 0.0f;
            uint32_t pk[64];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float p0 = ex2_approx(__uint_as_float(v[q][c]) - m_sub);
                    const float p1 = ex2_approx(__uint_as_float(v[q][c + 1]) - m_sub);
                    rs += p0 + p1;
                    pk[(q * 32 + c) >> 1] = pack_bf16x2(p0, p1);
                }
            l = fmaf(l, alpha, rs);
            m_run = m_use;

            // O and the P buffer are free once the previous PV has completed
            if (t > 0 && !mbar_wait(&bar_pv, (t - 1) & 1, wc, 0x209)) { ok = false; break; }
            tc_fence_after();
            if (t > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t o[32];
                    const uint32_t oa = tmem + t_lane + O_COL + q * 32;
                    tmem_ld32(oa, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                    tmem_st32(oa, o);
                }
                tmem_wait_st();
            }
            // P row r, keys 0..127, into the two 64-key swizzled chunks
#pragma unroll
            for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int base = ch * 32 + u * 4;
                    const uint4 val = make_uint4(pk[base], pk[base + 1], pk[base + 2], pk[base + 3]);
                    *reinterpret_cast<uint4 *>(sP + ch * 16384 + r * 128 + ((u ^ (r & 7)) << 4)) = val;
                }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_p);
        }
        // epilogue: O / l -> bf16
        if (ok && mbar_wait(&bar_pv, (ntiles - 1) & 1, wc, 0x20a)) {
            tc_fence_after();
            const float inv = l > 0.0f ? 1.0f / l : 0.0f;
            __nv_bfloat16 *orow = a.O + (tok0 + r) * D;
#pragma unroll
            for (int q = 0; q < D / 32; ++q) {
                uint32_t o[32];
                tmem_ld32(tmem + t_lane + O_COL + q * 32, o);
                tmem_wait_ld();
                if (r < nrows) {
#pragma unroll
                    for (int c = 0; c < 32; c += 8) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(o[c + 0]) * inv, __uint_as_float(o[c + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(o[c + 2]) * inv, __uint_as_float(o[c + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(o[c + 4]) * inv, __uint_as_float(o[c + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(o[c + 6]) * inv, __uint_as_float(o[c + 7]) * inv);
                        *reinterpret_cast<uint4 *>(orow + q * 32 + c) = w;
                    }
                }
            }
            if (a.lse && r < nrows) a.lse[tok0 + r] = (m_run + __log2f(l)) * kLn2;
        }
        tc_fence_before();
    }

    // ------------------------------ teardown --------------------------------------
    __syncthreads();
    if (abort_s) {
        if (warp == 0 && lane == 0) {
            for (int t = k_issued - kKStages > 0 ? k_issued - kKStages : 0; t < k_issued; ++t) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&bar_kf[t % kKStages], (t / kKStages) & 1) &&
                       globaltimer_ns() - t0 < a.wait_ns) {
                }
            }
            for (int t = v_issued - kVStages > 0 ? v_issued - kVStages : 0; t < v_issued; ++t) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&bar_vf[t % kVStages], (t / kVStages) & 1) &&
                       globaltimer_ns() - t0 < a.wait_ns) {
                }
            }
        }
        if (warp == 1 && lane == 0 && committed > 0) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&bar_pv, (committed - 1) & 1) && globaltimer_ns() - t0 < a.wait_ns) {
            }
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <int D, int BK>
cudaError_t launch_attn_t(const AttnArgs &a, const AttnMaps &maps, cudaStream_t stream) {
    const size_t smem = (1 + kKStages + kVStages) * (size_t)(128 * D * 2) + 128 * 128 * 2 + 1024;
    cudaError_t e = cudaFuncSetAttribute(gather_attn_kernel<D, BK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gather_attn_kernel<D, BK><<<(unsigned)a.rows, kAttnThreads, smem, stream>>>(maps, a);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_attn_d(const AttnArgs &a, const AttnMaps &maps, cudaStream_t stream) {
    switch (a.Bk) {
        case 16: return launch_attn_t<D, 16>(a, maps, stream);
        case 32: return launch_attn_t<D, 32>(a, maps, stream);
        case 64: return launch_attn_t<D, 64>(a, maps, stream);
        case 128: return launch_attn_t<D, 128>(a, maps, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_attention(const AttnArgs &a, const AttnMaps &maps, int, cudaStream_t stream) {
    if (a.rows < 1) return cudaSuccess;
    return a.D == 128 ? launch_attn_d<128>(a, maps, stream) : launch_attn_d<64>(a, maps, stream);
}

}  // namespace abatt
