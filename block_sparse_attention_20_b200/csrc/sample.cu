// sample.cu -- SIP: exact Poisson draw of key blocks with inclusion
// probabilities proportional to the IBCS estimates, compacted into ascending
// block lists with log-weights -ln(pi) ("Accurate Block Attention", abstract,
// sampling sentence: blocks are drawn in proportion to the estimates and
// re-weighted by the inverse inclusion probability).
//
// One CTA per row (query block).  Up to nK = 10240 the row's 48-bit
// fixed-point weights live in registers, each thread (256 or 512 per CTA)
// holding a contiguous run of at most 20 blocks (sample_compact_reg_kernel);
// beyond that they are built once into shared memory (sample_compact_kernel).  The water-filling
// rounds, the Philox draws and the ordered compaction run from there: four
// consecutive blocks share one Philox block (one draw each), and positions in
// the list come from a block-wide scan of the per-thread counts, so the list
// is ascending.  Every decision is integer
// arithmetic on the fixed-point weights: the result does not depend on the
// launch configuration.
#include "kernels.cuh"

namespace abatt {

namespace {

constexpr int kSampleThreads = 256;
constexpr int kSampleWarps = kSampleThreads / 32;
constexpr int kCacheMaxBlocks = 8192;  // weights cached in shared memory up to this nK

// round-half-even(p * 2^48) for p clamped to [0, 1] (NaN and negatives -> 0).
// The scaling by a power of two is exact in fp32 (subnormal inputs included:
// the build keeps subnormals), and the conversion to int64 rounds half to
// even, so this is the exact fixed-point value.
__device__ __forceinline__ int64_t to_fixed48(float p) {
    if (!(p > 0.0f)) return 0;
    if (p >= 1.0f) return int64_t(1) << 48;
    return __float2ll_rn(__fmul_rn(p, 0x1p48f));
}

// ceil(T / R) for 0 < T < 2^53, R > 0: the double quotient is within 1/16 of
// T / R (both operands are exact in double), so its ceiling is off by at most
// one, which the exact integer test corrects.
__device__ __forceinline__ int64_t ceil_div(int64_t T, int64_t R) {
    int64_t q = (int64_t)ceil((double)T / (double)R);
    if (q * R < T) ++q;
    else if ((q - 1) * R >= T) --q;
    return q;
}

// Philox4x32-10 (Salmon et al., SC 2011): ten rounds, published multipliers
// and Weyl increments.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
        const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c;
}

template <typename T>
__device__ __forceinline__ T block_sum(T v, T *scratch /*[kSampleWarps]*/) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();  // scratch reuse guard
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    T tot = 0;
#pragma unroll
    for (int w = 0; w < kSampleWarps; ++w) tot += scratch[w];
    return tot;
}

// U * T < (RP << 32), all unsigned, U < 2^32, T and RP < 2^63 (96-bit compare).
__device__ __forceinline__ bool draw_below(uint32_t U, uint64_t T, uint64_t RP) {
    const uint64_t lhs_lo = (uint64_t)U * T;
    const uint64_t lhs_hi = __umul64hi((uint64_t)U, T);
    const uint64_t rhs_lo = RP << 32;
    const uint64_t rhs_hi = RP >> 32;
    return lhs_hi < rhs_hi || (lhs_hi == rhs_hi && lhs_lo < rhs_lo);
}

template <bool CACHED>
__global__ void __launch_bounds__(kSampleThreads) sample_compact_kernel(SampleArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    // CACHED: int64 weights [nK_pad]; else fp32 p [nK_pad].  Then sat bytes [nK_pad].
    int64_t *Pw = reinterpret_cast<int64_t *>(smem_raw);
    float *ps = reinterpret_cast<float *>(smem_raw);
    uint8_t *sat = smem_raw + (CACHED ? 8 : 4) * (size_t)a.nK_pad;
    __shared__ int64_t red64[kSampleWarps];
    __shared__ int32_t wtot[kSampleWarps];

    const int nK = a.nK;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto weight = [&](int b) -> int64_t { return CACHED ? Pw[b] : to_fixed48(ps[b]); };

    for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
        const float *prow = a.p + row * (int64_t)nK;
        // eight loads in flight per thread before any is used
        for (int b0 = 0; b0 < nK; b0 += 8 * kSampleThreads) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int b = b0 + u * kSampleThreads + tid;
                v[u] = b < nK ? __ldg(prow + b) : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int b = b0 + u * kSampleThreads + tid;
                if (b < nK) {
                    if (CACHED) Pw[b] = to_fixed48(v[u]);
                    else ps[b] = v[u];
                    sat[b] = 0;
                }
            }
        }
        __syncthreads();

        const int i = (int)(row % a.nQ);
        const int64_t bh = row / a.nQ;
        const int h = (int)(bh % a.H);
        const int beta = (int)(bh / a.H);

        // ---- inclusion probabilities: exact water-filling ----------------
        int64_t R = a.M, T = 0;
        if (a.M >= nK) {
            for (int b = tid; b < nK; b += kSampleThreads) sat[b] = 1;
            R = 0;
        } else {
            // T = sum of the weights outside S; a round adds every b outside S
            // with R * P_b >= T, i.e. P_b >= ceil(T / R) (positive integers),
            // and carries T forward by subtracting what it added
            int64_t local = 0;
            for (int b = tid; b < nK; b += kSampleThreads) local += weight(b);
            T = block_sum<int64_t>(local, red64);
            int64_t in_s = 0;
            for (int round = 0; round <= nK; ++round) {
                R = a.M - in_s;
                if (T == 0 || R <= 0) break;
                const int64_t thr = ceil_div(T, R);
                int64_t added = 0, added_w = 0;
                for (int b = tid; b < nK; b += kSampleThreads) {
                    if (sat[b]) continue;
                    const int64_t w = weight(b);
                    if (w >= thr) {
                        sat[b] = 1;
                        ++added;
                        added_w += w;
                    }
                }
                added = block_sum<int64_t>(added, red64);
                if (added == 0) break;
                added_w = block_sum<int64_t>(added_w, red64);
                in_s += added;
                T -= added_w;
            }
        }
        __syncthreads();

        // ---- draws and ordered compaction: thread t owns blocks 4g..4g+3 --
        int32_t *idx_row = a.idx + row * (int64_t)a.capacity;
        float *logw_row = a.logw + row * (int64_t)a.capacity;
        int running = 0;
        for (int g0 = 0; 4 * g0 < nK; g0 += kSampleThreads) {
            const int g = g0 + tid;
            const int b0 = 4 * g;
            bool take[4] = {false, false, false, false};
            uint64_t rp[4] = {0, 0, 0, 0};
            int cnt = 0;
            if (b0 < nK) {
                const uint4 u = philox4x32_10(make_uint4((uint32_t)g, (uint32_t)(a.paired ? i >> 1 : i),
                                                         (uint32_t)h + a.h_off, (uint32_t)beta + a.b_off),
                                              a.key0, a.key1);
                const uint32_t U[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int b = b0 + k;
                    if (b >= nK) break;
                    if (sat[b]) {
                        take[k] = true;
                    } else {
                        rp[k] = (uint64_t)(R * weight(b));
                        take[k] = rp[k] != 0 && draw_below(U[k], (uint64_t)T, rp[k]);
                    }
                    cnt += take[k];
                }
            }
            // block-wide exclusive scan of the per-thread counts
            int x = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (lane == 31) wtot[warp] = x;
            __syncthreads();
            int pos = running + x - cnt, total = 0;
#pragma unroll
            for (int w = 0; w < kSampleWarps; ++w) {
                const int c = wtot[w];
                pos += w < warp ? c : 0;
                total += c;
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (!take[k]) continue;
                if (pos < a.capacity) {
                    idx_row[pos] = b0 + k;
                    logw_row[pos] =
                        rp[k] ? (float)(-log((double)(int64_t)rp[k] / (double)T)) : 0.0f;
                }
                ++pos;
            }
            running += total;
            __syncthreads();
        }
        if (tid == 0) {
            if (running > a.capacity) {
                raise_flag(a.status, ABATT_DEVFLAG_CAPACITY);
                running = a.capacity;
            }
            a.counts[row] = running;
        }
        __syncthreads();
    }
}

// Register-resident variant for nK <= 4*G*NT: thread t owns the contiguous
// run of blocks [t*4G, (t+1)*4G) (G Philox groups), its fixed-point weights
// stay in registers for every water-filling round, and one block-wide scan of
// the per-thread counts places the drawn blocks in ascending order.
template <int NT, int G>
__global__ void __launch_bounds__(NT, NT == 256 ? 4 : 1) sample_compact_reg_kernel(SampleArgs a) {
    constexpr int NW = NT / 32;
    constexpr int PER = 4 * G;  // blocks per thread (<= 32: the masks are 32-bit)
    // the row is staged through shared memory with coalesced loads; thread
    // runs are SP words apart, which keeps the 16-byte reads of eight
    // consecutive threads on distinct banks
    constexpr int SP = (PER % 8 == 4) ? PER : PER + 4;
    __shared__ __align__(16) float ps[NT * SP];
    __shared__ int64_t red_w[NW];
    __shared__ int32_t red_c[NW];
    __shared__ int32_t wtot[NW];
    __shared__ uint32_t sat_s[NT];  // saturation mask of each thread's run
    __shared__ int32_t hist_s[128];  // top-M: digit histogram of the radix select
    __shared__ int64_t sel_prefix_s;
    __shared__ int32_t sel_k_s;
    const int nK = a.nK;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b0 = tid * PER;

    for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
        const float *prow = a.p + row * (int64_t)nK;
        __syncthreads();  // the previous row is done with ps
#pragma unroll
        for (int u = 0; u < PER; u += 4) {
            float v[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int b = (u + q) * NT + tid;
                v[q] = b < nK ? __ldg(prow + b) : 0.0f;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int b = (u + q) * NT + tid;
                ps[(b / PER) * SP + b % PER] = v[q];
            }
        }
        __syncthreads();
        int64_t P[PER];
#pragma unroll
        for (int k = 0; k < PER; k += 4) {
            const float4 q = *reinterpret_cast<const float4 *>(ps + tid * SP + k);
            P[k] = to_fixed48(q.x);
            P[k + 1] = to_fixed48(q.y);
            P[k + 2] = to_fixed48(q.z);
            P[k + 3] = to_fixed48(q.w);
        }
        const int i = (int)(row % a.nQ);
        const int64_t bh = row / a.nQ;
        const int h = (int)(bh % a.H);
        const int beta = (int)(bh / a.H);
        const int nmine = max(0, min(PER, nK - b0));
        const uint32_t valid = nmine >= 32 ? 0xffffffffu : ((1u << nmine) - 1u);

        uint32_t sat = 0, take = 0;
        int64_t R = a.M, T = 0;
        if (a.topk) {
            // ---- top-M truncation: the M largest weights, ties to the lower index.
            // Radix select of the M-th largest key, seven 7-bit digits from the
            // top (keys are < 2^49), then the ties admitted in index order.
            if (a.M >= nK) {
                take = valid;
            } else if (a.M > 0) {
                int64_t prefix = 0, mask = 0;
                int k = (int)a.M;  // rank still to find among the candidates, 1 = largest
                for (int dgt = 6; dgt >= 0; --dgt) {
                    const int sh = 7 * dgt;
                    if (tid < 128) hist_s[tid] = 0;
                    __syncthreads();
#pragma unroll
                    for (int q = 0; q < PER; ++q)
                        if (((valid >> q) & 1u) && (P[q] & mask) == prefix)
                            atomicAdd(&hist_s[(int)((P[q] >> sh) & 127)], 1);
                    __syncthreads();
                    if (warp == 0) {
                        // lane l holds bins 4l..4l+3; counts at or above each bin by a
                        // suffix scan over the lanes, from the largest digit down
                        int c[4], sum = 0;
#pragma unroll
                        for (int u = 0; u < 4; ++u) { c[u] = hist_s[4 * lane + u]; sum += c[u]; }
                        int suf = sum;  // inclusive suffix over lanes l..31
#pragma unroll
                        for (int o = 1; o < 32; o <<= 1) {
                            const int y = __shfl_down_sync(0xffffffffu, suf, o);
                            if (lane + o < 32) suf += y;
                        }
                        int above = suf - sum;  // keys in bins of higher lanes
                        int found = -1, above_found = 0;
#pragma unroll
                        for (int u = 3; u >= 0; --u) {
                            if (found < 0 && above < k && above + c[u] >= k) {
                                found = 4 * lane + u;
                                above_found = above;
                            }
                            above += c[u];
                        }
                        const uint32_t who = __ballot_sync(0xffffffffu, found >= 0);
                        const int src = __ffs(who) - 1;
                        const int v = __shfl_sync(0xffffffffu, found, src);
                        const int ab = __shfl_sync(0xffffffffu, above_found, src);
                        if (lane == 0) {
                            sel_prefix_s = prefix | ((int64_t)v << sh);
                            sel_k_s = k - ab;
                        }
                    }
                    __syncthreads();
                    prefix = sel_prefix_s;
                    k = sel_k_s;
                    mask |= (int64_t)127 << sh;
                    __syncthreads();  // hist_s and the selection are reused next digit
                }
                // prefix is the M-th largest key; k of the keys equal to it are kept,
                // the first k by index: an exclusive scan of the per-thread tie counts
                uint32_t ties = 0;
#pragma unroll
                for (int q = 0; q < PER; ++q) {
                    if (!((valid >> q) & 1u)) continue;
                    if (P[q] > prefix) take |= 1u << q;
                    else if (P[q] == prefix) ties |= 1u << q;
                }
                const int tc = __popc(ties);
                int x = tc;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o) x += y;
                }
                if (lane == 31) wtot[warp] = x;
                __syncthreads();
                int before = x - tc;
#pragma unroll
                for (int q = 0; q < NW; ++q) before += q < warp ? wtot[q] : 0;
                __syncthreads();  // wtot is reused by the compaction
#pragma unroll
                for (int q = 0; q < PER; ++q)
                    if (((ties >> q) & 1u) && before++ < k) take |= 1u << q;
            }
            sat = take;  // kept blocks carry log-weight 0
        } else {
        // ---- inclusion probabilities: exact water-filling (as in the shared-memory kernel)
        if (a.M >= nK) {
            sat = valid;
            R = 0;
        } else {
            int64_t local = 0;
#pragma unroll
            for (int k = 0; k < PER; ++k) local += P[k];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) local += __shfl_down_sync(0xffffffffu, local, o);
            if (lane == 0) red_w[warp] = local;
            __syncthreads();
#pragma unroll
            for (int q = 0; q < NW; ++q) T += red_w[q];
            int64_t in_s = 0;
            // the largest weight of this thread's run still outside S: a round
            // with a higher threshold adds nothing here
            int64_t wmax = 0;
#pragma unroll
            for (int k = 0; k < PER; ++k) wmax = max(wmax, P[k]);
            for (int round = 0; round <= nK; ++round) {
                R = a.M - in_s;
                if (T == 0 || R <= 0) break;
                const int64_t thr = ceil_div(T, R);
                int cnt = 0;
                int64_t w = 0;
                if (wmax >= thr) {
                    int64_t rest = 0;
#pragma unroll
                    for (int k = 0; k < PER; ++k) {
                        if ((sat >> k) & 1u) continue;
                        if (P[k] >= thr) {
                            sat |= 1u << k;
                            ++cnt;
                            w += P[k];
                        } else {
                            rest = max(rest, P[k]);
                        }
                    }
                    wmax = rest;
                }
                // count and weight reduced together: one barrier pair per round
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    cnt += __shfl_down_sync(0xffffffffu, cnt, o);
                    w += __shfl_down_sync(0xffffffffu, w, o);
                }
                __syncthreads();
                if (lane == 0) {
                    red_c[warp] = cnt;
                    red_w[warp] = w;
                }
                __syncthreads();
                int added = 0;
                int64_t added_w = 0;
#pragma unroll
                for (int q = 0; q < NW; ++q) {
                    added += red_c[q];
                    added_w += red_w[q];
                }
                if (added == 0) break;
                in_s += added;
                T -= added_w;
            }
        }
        sat &= valid;

        // ---- draws: group g = tid*G + u gives blocks 4g..4g+3 ----------------
#pragma unroll
        for (int u = 0; u < G; ++u) {
            const int g = tid * G + u;
            if (4 * g >= nK) break;
            const uint4 r4 =
                philox4x32_10(make_uint4((uint32_t)g, (uint32_t)(a.paired ? i >> 1 : i), (uint32_t)h + a.h_off,
                                         (uint32_t)beta + a.b_off),
                              a.key0, a.key1);
            const uint32_t U[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int bit = 4 * u + k;
                if (!((valid >> bit) & 1u)) continue;
                if ((sat >> bit) & 1u) {
                    take |= 1u << bit;
                } else {
                    const uint64_t rp = (uint64_t)(R * P[bit]);
                    if (rp != 0 && draw_below(U[k], (uint64_t)T, rp)) take |= 1u << bit;
                }
            }
        }
        }  // SIP
        // ---- ordered compaction: exclusive scan of the per-thread counts -------
        const int cnt = __popc(take);
        int x = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        __syncthreads();  // wtot reuse guard
        if (lane == 31) wtot[warp] = x;
        __syncthreads();
        int pos = x - cnt, total = 0;
#pragma unroll
        for (int q = 0; q < NW; ++q) {
            const int c = wtot[q];
            pos += q < warp ? c : 0;
            total += c;
        }
        int32_t *idx_row = a.idx + row * (int64_t)a.capacity;
        float *logw_row = a.logw + row * (int64_t)a.capacity;
        // static indices keep P in registers
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            if (!((take >> k) & 1u)) continue;
            if (pos < a.capacity) idx_row[pos] = b0 + k;
            ++pos;
        }
        sat_s[tid] = sat;
        const int n = min(total, a.capacity);
        if (tid == 0) {
            if (total > a.capacity) raise_flag(a.status, ABATT_DEVFLAG_CAPACITY);
            a.counts[row] = n;
        }
        __syncthreads();  // the list and the saturation masks are complete
        // log-weights in a second, convergent pass: list entry j on thread
        // j mod NT, its weight re-derived from the staged row
        for (int j = tid; j < n; j += NT) {
            const int b = idx_row[j];
            const int owner = b / PER, k = b - owner * PER;
            float lw = 0.0f;
            if (!((sat_s[owner] >> k) & 1u)) {
                const int64_t rp = R * to_fixed48(ps[owner * SP + k]);
                lw = (float)(-log((double)rp / (double)T));
            }
            logw_row[j] = lw;
        }
    }
}

}  // namespace

size_t sample_smem_bytes(int nK) {
    const size_t nK_pad = (size_t)((nK + 3) & ~3);
    return (nK <= kCacheMaxBlocks ? 8 : 4) * nK_pad + nK_pad;
}

cudaError_t launch_sample(const SampleArgs &a, int num_sms, cudaStream_t stream) {
    int64_t grid = a.rows;
    if (grid < 1) return cudaSuccess;
    // register-resident kernel: at most five Philox groups (20 blocks) per
    // thread, with 256 threads up to nK = 5120 and 512 up to 10240
    const int G256 = (a.nK + 1023) / 1024, G512 = (a.nK + 2047) / 2048;
    if (G256 <= 5 || G512 <= 5) {
        const int64_t cap = (int64_t)num_sms * (G256 <= 5 ? 8 : 4);
        if (grid > cap) grid = cap;
        const unsigned gr = (unsigned)grid;
        if (G256 <= 5) {
            switch (G256) {
                case 1: sample_compact_reg_kernel<256, 1><<<gr, 256, 0, stream>>>(a); break;
                case 2: sample_compact_reg_kernel<256, 2><<<gr, 256, 0, stream>>>(a); break;
                case 3: sample_compact_reg_kernel<256, 3><<<gr, 256, 0, stream>>>(a); break;
                case 4: sample_compact_reg_kernel<256, 4><<<gr, 256, 0, stream>>>(a); break;
                default: sample_compact_reg_kernel<256, 5><<<gr, 256, 0, stream>>>(a); break;
            }
        } else if (G512 <= 3) {
            sample_compact_reg_kernel<512, 3><<<gr, 512, 0, stream>>>(a);
        } else if (G512 == 4) {
            sample_compact_reg_kernel<512, 4><<<gr, 512, 0, stream>>>(a);
        } else {
            sample_compact_reg_kernel<512, 5><<<gr, 512, 0, stream>>>(a);
        }
        return cudaGetLastError();
    }
    const size_t smem = sample_smem_bytes(a.nK);
    const int64_t cap = (int64_t)num_sms * 64;
    if (grid > cap) grid = cap;
    cudaError_t e;
    if (a.nK <= kCacheMaxBlocks) {
        e = cudaFuncSetAttribute(sample_compact_kernel<true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        sample_compact_kernel<true><<<(unsigned)grid, kSampleThreads, smem, stream>>>(a);
    } else {
        e = cudaFuncSetAttribute(sample_compact_kernel<false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        sample_compact_kernel<false><<<(unsigned)grid, kSampleThreads, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace abatt
