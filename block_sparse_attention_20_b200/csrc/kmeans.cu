// kmeans.cu -- IBCS part 1: Lloyd k-means of the queries of every query block,
// on the block's own tokens and in their original order ("Accurate Block
// Attention", abstract, selector sentence: queries are clustered only within
// each query block, without permuting tokens).
//
// One CTA of 128 threads per query block; thread r owns query row r.  The
// block's queries sit in shared memory as fp32, transposed with a padded
// stride so both the per-row distance loop and the per-dimension centroid
// sums read conflict-free.  Rounds are deterministic: the centroid update
// sums each cluster's rows in ascending row order (a stable counting sort by
// cluster, built from warp ballots).
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

template <int D>
__global__ void __launch_bounds__(kKmThreads) kmeans_qblock_kernel(KmeansArgs a) {
    constexpr int LD = 129;  // padded row stride of the transposed block
    extern __shared__ __align__(16) float km_smem[];
    float *qT = km_smem;                     // [D][LD]
    float *cent = qT + D * LD;               // [kMaxC][D]
    __shared__ int assign_s[128];
    __shared__ int order_s[128];
    __shared__ uint32_t mask_s[4][kMaxC];
    __shared__ int cnt_s[kMaxC];
    __shared__ int base_s[kMaxC];
    __shared__ int woff_s[4][kMaxC];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int C = a.C;

    for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
        const int i = (int)(row % a.nQ);
        const int64_t bh = row / a.nQ;
        const int n = min(128, a.N - i * 128);
        const int ce = min(C, n);
        const __nv_bfloat16 *qblk = a.Q + (bh * (int64_t)a.N + (int64_t)i * 128) * D;

        // load the block (thread r <- row r), transposed into qT[x][r]
        if (tid < n) {
            const uint4 *src = reinterpret_cast<const uint4 *>(qblk + (int64_t)tid * D);
#pragma unroll 4
            for (int v = 0; v < D / 8; ++v) {
                uint4 u = src[v];
                const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&u);
#pragma unroll
                for (int k = 0; k < 8; ++k) qT[(v * 8 + k) * LD + tid] = __bfloat162float(e[k]);
            }
        }
        __syncthreads();
        for (int e = tid; e < kMaxC * D; e += kKmThreads) {
            const int j = e / D, x = e % D;
            cent[e] = j < ce ? qT[x * LD + (int)(((int64_t)j * n) / ce)] : 0.0f;
        }
        __syncthreads();

        const int rounds = a.iters > 0 ? a.iters : 1;
        for (int it = 0; it < rounds; ++it) {
            // ---- assignment ----
            int best = -1;
            if (tid < n) {
                float acc[kMaxC];
#pragma unroll
                for (int j = 0; j < kMaxC; ++j) acc[j] = 0.0f;
#pragma unroll 4
                for (int x = 0; x < D; ++x) {
                    const float q = qT[x * LD + tid];
#pragma unroll
                    for (int j = 0; j < kMaxC; ++j) {
                        if (j < ce) {
                            const float df = q - cent[j * D + x];
                            acc[j] = fmaf(df, df, acc[j]);
                        }
                    }
                }
                float bd = acc[0];
                best = 0;
#pragma unroll
                for (int j = 1; j < kMaxC; ++j)
                    if (j < ce && acc[j] < bd) {
                        bd = acc[j];
                        best = j;
                    }
            }
            assign_s[tid] = best;
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
                    float s = 0.0f;
                    const int b0 = base_s[j];
                    for (int e = 0; e < c; ++e) s += qT[x * LD + order_s[b0 + e]];
                    cent[j * D + x] = s / (float)c;
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

size_t kmeans_smem_bytes(int D) { return sizeof(float) * (size_t)(D * 129 + kMaxC * D); }

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
