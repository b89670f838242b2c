// sample.cu -- SIP: exact Poisson draw of key blocks with inclusion
// probabilities proportional to the IBCS estimates, compacted into ascending
// block lists with log-weights -ln(pi) ("Accurate Block Attention", abstract,
// sampling sentence: blocks are drawn in proportion to the estimates and
// re-weighted by the inverse inclusion probability).
//
// One CTA per row (query block).  The row's probabilities stay in shared
// memory; the water-filling rounds, the Philox draws and the ordered
// compaction (warp ballot + block prefix sum) all run from there.  Every
// decision is integer arithmetic on 48-bit fixed-point weights, so the
// result does not depend on the launch configuration.
#include "kernels.cuh"

namespace abatt {

namespace {

constexpr int kSampleThreads = 256;
constexpr int kSampleWarps = kSampleThreads / 32;

__device__ __forceinline__ int64_t to_fixed48(float p) {
    // p * 2^48 is exact in fp32 (a power-of-two scaling of a value in [0, 1]);
    // the conversion rounds half to even.
    if (!(p > 0.0f)) return 0;  // zero, negative, NaN
    if (p > 1.0f) p = 1.0f;
    return __float2ll_rn(p * 281474976710656.0f);
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

__global__ void __launch_bounds__(kSampleThreads)
    sample_compact_kernel(SampleArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *ps = reinterpret_cast<float *>(smem_raw);                         // [nK]
    uint8_t *sat = reinterpret_cast<uint8_t *>(smem_raw + sizeof(float) * a.nK_pad);  // [nK]
    __shared__ int64_t red64[kSampleWarps];
    __shared__ int32_t wcount[kSampleWarps];

    const int nK = a.nK;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
        const float *prow = a.p + row * (int64_t)nK;
        for (int b = tid; b < nK; b += kSampleThreads) {
            ps[b] = prow[b];
            sat[b] = 0;
        }
        __syncthreads();

        const int i = (int)(row % a.nQ);
        const int64_t bh = row / a.nQ;
        const int h = (int)(bh % a.H);
        const int beta = (int)(bh / a.H);

        // ---- inclusion probabilities: exact water-filling ----------------
        int64_t R = a.M, T = 0;
        const bool keep_all = a.M >= nK;
        if (keep_all) {
            for (int b = tid; b < nK; b += kSampleThreads) sat[b] = 1;
            R = 0;
        } else {
            int64_t in_s = 0;
            for (int round = 0; round <= nK; ++round) {
                R = a.M - in_s;
                int64_t local = 0;
                for (int b = tid; b < nK; b += kSampleThreads)
                    if (!sat[b]) local += to_fixed48(ps[b]);
                T = block_sum<int64_t>(local, red64);
                if (T == 0 || R <= 0) break;
                int64_t added = 0;
                for (int b = tid; b < nK; b += kSampleThreads) {
                    if (!sat[b] && R * to_fixed48(ps[b]) >= T) {
                        sat[b] = 1;
                        ++added;
                    }
                }
                added = block_sum<int64_t>(added, red64);
                if (added == 0) break;
                in_s += added;
            }
        }
        __syncthreads();

        // ---- draws and ordered compaction -------------------------------
        int32_t *idx_row = a.idx + row * (int64_t)a.capacity;
        float *logw_row = a.logw + row * (int64_t)a.capacity;
        int running = 0;
        for (int base = 0; base < nK; base += kSampleThreads) {
            const int b = base + tid;
            bool take = false;
            float lw = 0.0f;
            if (b < nK) {
                if (sat[b]) {
                    take = true;
                } else {
                    const uint64_t RP = (uint64_t)(R * to_fixed48(ps[b]));
                    if (RP != 0) {
                        const uint4 u = philox4x32_10(
                            make_uint4((uint32_t)(b >> 2), (uint32_t)i, (uint32_t)h, (uint32_t)beta),
                            a.key0, a.key1);
                        const int w = b & 3;
                        const uint32_t U = w == 0 ? u.x : w == 1 ? u.y : w == 2 ? u.z : u.w;
                        take = draw_below(U, (uint64_t)T, RP);
                        if (take) {
                            const double x = (double)(int64_t)RP / (double)T;
                            lw = (float)(-log(x));
                        }
                    }
                }
            }
            const uint32_t ballot = __ballot_sync(0xffffffffu, take);
            if (lane == 0) wcount[warp] = __popc(ballot);
            __syncthreads();
            int before = 0, total = 0;
#pragma unroll
            for (int w = 0; w < kSampleWarps; ++w) {
                const int c = wcount[w];
                before += w < warp ? c : 0;
                total += c;
            }
            if (take) {
                const int pos = running + before + __popc(ballot & ((1u << lane) - 1u));
                if (pos < a.capacity) {
                    idx_row[pos] = b;
                    logw_row[pos] = lw;
                }
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

}  // namespace

size_t sample_smem_bytes(int nK) {
    const int nK_pad = (nK + 3) & ~3;
    return sizeof(float) * (size_t)nK_pad + (size_t)nK_pad;
}

cudaError_t launch_sample(const SampleArgs &a, int num_sms, cudaStream_t stream) {
    const size_t smem = sample_smem_bytes(a.nK);
    cudaError_t e = cudaFuncSetAttribute(sample_compact_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int64_t grid = a.rows;
    const int64_t cap = (int64_t)num_sms * 16;
    if (grid > cap) grid = cap;
    if (grid < 1) return cudaSuccess;
    sample_compact_kernel<<<(unsigned)grid, kSampleThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace abatt
