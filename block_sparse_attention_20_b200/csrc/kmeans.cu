// kmeans.cu -- IBCS part 1: Lloyd k-means of the queries of every query block,
// on the block's own tokens and in their original order ("Accurate Block
// Attention", abstract, selector sentence: queries are clustered only within
// each query block, without permuting tokens).
//
// One CTA of 128 threads (4 warps) per query block.  The block's queries stay
// in shared memory as bf16 (exact copies of the inputs).  Per round:
//   - distances: ||c_j||^2 - 2 q.c_j, the dot products on the tensor cores
//     (mma.sync m16n8k16, bf16 in, fp32 accumulate) with each fp32 centroid
//     split into a bf16 high part and a bf16 residual, so the products carry
//     about 16 significant bits of the centroid; warp w takes rows
//     32w..32w+31; the argmin (ties to the lower index) is reduced across the
//     four lanes that share a row;
//   - update: a stable counting sort of the rows by cluster (warp ballots),
//     then thread x sums dimension x of each cluster's rows as four
//     interleaved partial sums in ascending row order, combined in a fixed
//     order (deterministic), centroid = sum / size.
//
// Rules (open in the abstract, fixed here): C_eff = min(C, n) clusters;
// centroid j starts at row floor(j*n/C_eff); squared Euclidean distance,
// ties to the lower index; an empty cluster keeps its centroid; cluster
// sizes come from the last round's assignment.
//
// Outputs: scaled centroids split into bf16 hi + lo parts (the scoring GEMM
// operand, pre-multiplied by scale*log2(e) so the GEMM yields base-2
// logits), the cluster weights n_j/n, and optionally the fp32 centroids and
// cluster sizes.
#include "kernels.cuh"

namespace abatt {

namespace {

constexpr int kKmThreads = 128;
constexpr int kMaxC = 16;

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
__global__ void __launch_bounds__(kKmThreads) kmeans_qblock_kernel(KmeansArgs a) {
    constexpr int LDQ = D + 8;  // bf16 row stride: 4*row + column-pair spreads the banks
    extern __shared__ __align__(16) unsigned char km_smem[];
    __nv_bfloat16 *qs = reinterpret_cast<__nv_bfloat16 *>(km_smem);             // [128][LDQ]
    float *cent = reinterpret_cast<float *>(km_smem + 128 * LDQ * 2);            // [kMaxC][D]
    __nv_bfloat16 *chi = reinterpret_cast<__nv_bfloat16 *>(cent + kMaxC * D);    // [kMaxC][LDQ]
    __nv_bfloat16 *clo = chi + kMaxC * LDQ;                                      // [kMaxC][LDQ]
    __shared__ float cnorm[kMaxC];
    __shared__ int assign_s[128];
    __shared__ int order_s[128];
    __shared__ uint32_t mask_s[4][kMaxC];
    __shared__ int cnt_s[kMaxC];
    __shared__ int base_s[kMaxC];
    __shared__ int woff_s[4][kMaxC];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, cq = lane & 3;  // mma fragment coordinates
    const int C = a.C;
    const uint32_t *qw = reinterpret_cast<const uint32_t *>(qs);
    const uint32_t *hw = reinterpret_cast<const uint32_t *>(chi);
    const uint32_t *lw = reinterpret_cast<const uint32_t *>(clo);
    constexpr int LDW = LDQ / 2;  // row stride in 32-bit words

    for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
        const int i = (int)(row % a.nQ);
        const int64_t bh = row / a.nQ;
        const int n = min(128, a.N - i * 128);
        const int ce = min(C, n);
        const __nv_bfloat16 *qblk = a.Q + (bh * (int64_t)a.N + (int64_t)i * 128) * D;

        // the block's queries, row r by thread r; missing rows are zero
        {
            const uint4 *src = reinterpret_cast<const uint4 *>(qblk + (int64_t)tid * D);
            uint4 *dst = reinterpret_cast<uint4 *>(qs + tid * LDQ);
#pragma unroll 4
            for (int v = 0; v < D / 8; ++v) dst[v] = tid < n ? src[v] : make_uint4(0, 0, 0, 0);
        }
        __syncthreads();
        for (int e = tid; e < kMaxC * D; e += kKmThreads) {
            const int j = e / D, x = e % D;
            cent[e] = j < ce ? __bfloat162float(qs[(int)(((int64_t)j * n) / ce) * LDQ + x]) : 0.0f;
        }
        __syncthreads();

        const int rounds = a.iters > 0 ? a.iters : 1;
        for (int it = 0; it < rounds; ++it) {
            // ---- centroid operands: bf16 hi + lo, squared norms ----
            for (int e = tid; e < kMaxC * D; e += kKmThreads) {
                const int j = e / D, x = e % D;
                const float c = cent[e];
                const __nv_bfloat16 h = __float2bfloat16_rn(c);
                chi[j * LDQ + x] = h;
                clo[j * LDQ + x] = __float2bfloat16_rn(c - __bfloat162float(h));
            }
            // squared norms: warp w takes centroids w, w+4, ...; lanes split the dimensions
            for (int j = warp; j < kMaxC; j += 4) {
                float s = 0.0f;
#pragma unroll
                for (int x = lane; x < D; x += 32) s = fmaf(cent[j * D + x], cent[j * D + x], s);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                if (lane == 0) cnorm[j] = s;
            }
            __syncthreads();

            // ---- assignment: q.c on tensor cores, argmin over centroids ----
            const int nt = (ce + 7) >> 3;  // 8-wide centroid tiles
            float bestd[2][2];
            int besti[2][2];
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int r0 = warp * 32 + m * 16;
#pragma unroll
                for (int h = 0; h < 2; ++h) { bestd[m][h] = __int_as_float(0x7f800000); besti[m][h] = 0; }
                for (int t = 0; t < nt; ++t) {
                    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                    for (int k0 = 0; k0 < D; k0 += 16) {
                        const int kw = (k0 >> 1) + cq;  // word of column pair k0 + 2cq
                        uint32_t af[4];
                        af[0] = qw[(r0 + g) * LDW + kw];
                        af[1] = qw[(r0 + g + 8) * LDW + kw];
                        af[2] = qw[(r0 + g) * LDW + kw + 4];
                        af[3] = qw[(r0 + g + 8) * LDW + kw + 4];
                        const int cj = t * 8 + g;
                        mma_bf16_16816(acc, af, hw[cj * LDW + kw], hw[cj * LDW + kw + 4]);
                        mma_bf16_16816(acc, af, lw[cj * LDW + kw], lw[cj * LDW + kw + 4]);
                    }
                    // acc[0..1]: row g, centroids t*8+2cq+{0,1}; acc[2..3]: row g+8
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int j = t * 8 + 2 * cq + u;
                            const float dj = j < ce ? fmaf(-2.0f, acc[2 * h + u], cnorm[j])
                                                    : __int_as_float(0x7f800000);
                            if (dj < bestd[m][h]) { bestd[m][h] = dj; besti[m][h] = j; }
                        }
                }
                // combine the four lanes of each row (ties to the lower index)
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int o = 1; o < 4; o <<= 1) {
                        const float od = __shfl_xor_sync(0xffffffffu, bestd[m][h], o);
                        const int oi = __shfl_xor_sync(0xffffffffu, besti[m][h], o);
                        if (od < bestd[m][h] || (od == bestd[m][h] && oi < besti[m][h])) {
                            bestd[m][h] = od;
                            besti[m][h] = oi;
                        }
                    }
                if (cq == 0) {
                    assign_s[r0 + g] = (r0 + g) < n ? besti[m][0] : -1;
                    assign_s[r0 + g + 8] = (r0 + g + 8) < n ? besti[m][1] : -1;
                }
            }
            __syncthreads();
            const int best = assign_s[tid];

            // ---- stable counting sort of rows by cluster ----
            for (int j = 0; j < ce; ++j) {
                const uint32_t m = __ballot_sync(0xffffffffu, best == j);
                if (lane == 0) mask_s[warp][j] = m;
            }
            __syncthreads();
            if (tid == 0) {
                int acc = 0;
                for (int j = 0; j < ce; ++j) {
                    base_s[j] = acc;
                    for (int w = 0; w < 4; ++w) {
                        woff_s[w][j] = acc - base_s[j];
                        acc += __popc(mask_s[w][j]);
                    }
                    cnt_s[j] = acc - base_s[j];
                }
            }
            __syncthreads();
            if (best >= 0) {
                const int pos = base_s[best] + woff_s[warp][best] +
                                __popc(mask_s[warp][best] & ((1u << lane) - 1u));
                order_s[pos] = tid;
            }
            __syncthreads();
            if (a.iters == 0) break;  // sizes from the seeds, no update
            // ---- update: thread x sums dimension x of every cluster ----
            for (int x = tid; x < D; x += kKmThreads) {
                for (int j = 0; j < ce; ++j) {
                    const int c = cnt_s[j];
                    if (c == 0) continue;
                    // four interleaved partial sums (rows e = 0,4,8,.. / 1,5,9,.. / ...)
                    // in ascending row order each, combined in a fixed order
                    float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
                    const int b0 = base_s[j];
                    int e = 0;
                    for (; e + 4 <= c; e += 4) {
                        s0 += __bfloat162float(qs[order_s[b0 + e] * LDQ + x]);
                        s1 += __bfloat162float(qs[order_s[b0 + e + 1] * LDQ + x]);
                        s2 += __bfloat162float(qs[order_s[b0 + e + 2] * LDQ + x]);
                        s3 += __bfloat162float(qs[order_s[b0 + e + 3] * LDQ + x]);
                    }
                    if (e < c) s0 += __bfloat162float(qs[order_s[b0 + e] * LDQ + x]);
                    if (e + 1 < c) s1 += __bfloat162float(qs[order_s[b0 + e + 1] * LDQ + x]);
                    if (e + 2 < c) s2 += __bfloat162float(qs[order_s[b0 + e + 2] * LDQ + x]);
                    cent[j * D + x] = ((s0 + s1) + (s2 + s3)) / (float)c;
                }
            }
            __syncthreads();
        }

        // ---- outputs ----
        const float mul = a.logit_mul;  // scale * log2(e)
        for (int e = tid; e < C * D; e += kKmThreads) {
            const int j = e / D, x = e % D;
            const float c = j < ce ? cent[j * D + x] : 0.0f;
            const float v = c * mul;
            const __nv_bfloat16 hi = __float2bfloat16_rn(v);
            const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
            const int64_t o = (row * C + j) * (int64_t)D + x;
            a.cent_hi[o] = hi;
            a.cent_lo[o] = lo;
            if (a.cent_out) a.cent_out[o] = c;
        }
        if (tid < C) {
            const int c = tid < ce ? cnt_s[tid] : 0;
            a.weight[row * C + tid] = (float)c / (float)n;
            if (a.sizes_out) a.sizes_out[row * C + tid] = c;
        }
        __syncthreads();
    }
}

}  // namespace

size_t kmeans_smem_bytes(int D) {
    const int ldq = D + 8;
    return (size_t)128 * ldq * 2 + sizeof(float) * kMaxC * D + 2 * (size_t)kMaxC * ldq * 2;
}

cudaError_t launch_kmeans(const KmeansArgs &a, int num_sms, cudaStream_t stream) {
    int64_t grid = a.rows;
    const int64_t cap = (int64_t)num_sms * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) return cudaSuccess;
    const size_t smem = kmeans_smem_bytes(a.D);
    cudaError_t e;
    if (a.D == 128) {
        e = cudaFuncSetAttribute(kmeans_qblock_kernel<128>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kmeans_qblock_kernel<128><<<(unsigned)grid, kKmThreads, smem, stream>>>(a);
    } else {
        e = cudaFuncSetAttribute(kmeans_qblock_kernel<64>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kmeans_qblock_kernel<64><<<(unsigned)grid, kKmThreads, smem, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace abatt
