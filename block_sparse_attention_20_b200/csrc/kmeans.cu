// kmeans.cu -- IBCS part 1: Lloyd k-means of the queries of every query block,
// on the block's own tokens and in their original order ("Accurate Block
// Attention", abstract, selector sentence: queries are clustered only within
// each query block, without permuting tokens).
//
// One CTA of 128 threads (4 warps) per query block.  The block's queries stay
// in shared memory as bf16 (exact copies of the inputs).  Per round:
//   - distances: ||c_j||^2 - 2 q.c_j, the dot products on the tensor cores
//     (mma.sync m16n8k16, bf16 in, fp32 accumulate; fragments by ldmatrix,
//     the centroids' shared by a warp's two 16-row tiles; eight independent
//     accumulation chains) with each fp32 centroid
//     split into a bf16 high part and a bf16 residual, so the products carry
//     about 16 significant bits of the centroid; warp w takes rows
//     32w..32w+31; the argmin (ties to the lower index) is reduced across the
//     four lanes that share a row;
//   - update: cluster sizes from warp ballots (each warp counts its own 32
//     rows right after assigning them); the per-cluster sums of the
//     rows are one more tensor-core product, onehot(assignment)^T . Q
//     (16 x 128 times 128 x D, exact products, fp32 accumulation in a fixed
//     order, so the result is deterministic); centroid = sum * (1/size),
//     written with its bf16 operand parts, and each warp leaves the squared
//     norm of its quarter of the dimensions for the next assignment (two
//     block-wide barriers per round).
//
// Rules (open in the abstract, fixed here): C_eff = min(C, n) clusters;
// centroid j starts at row floor(j*n/C_eff); squared Euclidean distance,
// ties to the lower index; an empty cluster keeps its centroid; cluster
// sizes come from the last round's assignment.
//
// Outputs: the centroids pre-multiplied by scale*log2(e) and rounded to fp16
// (the scoring GEMM operand, so the GEMM yields base-2 logits), the cluster
// weights n_j/n, and optionally the fp32 centroids and cluster sizes.
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

// four 8x8 b16 matrices, transposed on the way: lane l supplies the address
// of row l%8 of matrix l/8
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void *row_addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(row_addr)));
}

// four 8x8 b16 matrices as stored: lane l supplies the address of row l%8
// of matrix l/8
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *row_addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(row_addr)));
}

// bf16 pair (lo, hi) of two 0/1 flags
__device__ __forceinline__ uint32_t onehot_pair(bool lo, bool hi) {
    return (lo ? 0x3F80u : 0u) | (hi ? 0x3F800000u : 0u);
}

template <int D>
__global__ void __launch_bounds__(kKmThreads, 5) kmeans_qblock_kernel(KmeansArgs a) {
    constexpr int LDQ = D + 8;  // bf16 row stride: 4*row + column-pair spreads the banks
    const int C = a.C;
    const int CP = C <= 8 ? 8 : 16;  // centroid rows held (one or two 8-wide MMA tiles)
    extern __shared__ __align__(16) unsigned char km_smem[];
    __nv_bfloat16 *qs = reinterpret_cast<__nv_bfloat16 *>(km_smem);             // [128][LDQ]
    float *cent = reinterpret_cast<float *>(km_smem + 128 * LDQ * 2);            // [CP][D]
    __nv_bfloat16 *chi = reinterpret_cast<__nv_bfloat16 *>(cent + CP * D);       // [CP][LDQ]
    __nv_bfloat16 *clo = chi + CP * LDQ;                                         // [CP][LDQ]
    __shared__ float cnp_s[4][kMaxC];  // squared centroid norms, partial per warp (dimension quarter)
    __shared__ int assign_s[128];
    __shared__ int wcnt_s[4][kMaxC];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, cq = lane & 3;  // mma fragment coordinates

    for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
        const int i = (int)(row % a.nQ);
        const int64_t bh = row / a.nQ;
        const int n = min(128, a.N - i * 128);
        const int ce = min(C, n);
        const __nv_bfloat16 *qblk = a.Q + a.st.head_base(bh) + (int64_t)i * 128 * a.st.sT;

        // the block's queries (each row's 16-byte chunks coalesced; rows sT
        // apart), copied straight into shared memory so all of a thread's
        // copies are in flight at once; missing rows are zero-filled
        {
            constexpr int CPR = D / 8;  // 16-byte chunks per row
#pragma unroll
            for (int c = tid; c < 128 * CPR; c += kKmThreads) {
                const int r = c / CPR, x8 = c % CPR;
                cp_async16_zfill(qs + r * LDQ + x8 * 8,
                                 reinterpret_cast<const uint4 *>(qblk + (int64_t)(r < n ? r : 0) * a.st.sT) + x8,
                                 r < n);
            }
            cp_async_wait_all();
        }
        __syncthreads();
        // a centroid coordinate and its tensor-core operands: bf16 high part and
        // bf16 residual
        auto put = [&](int j, int x, float c) {
            cent[j * D + x] = c;
            const __nv_bfloat16 h = __float2bfloat16_rn(c);
            chi[j * LDQ + x] = h;
            clo[j * LDQ + x] = __float2bfloat16_rn(c - __bfloat162float(h));
        };
        for (int e = tid; e < CP * D; e += kKmThreads) {
            const int j = e / D, x = e % D;
            put(j, x, j < ce ? __bfloat162float(qs[(j * n) / ce * LDQ + x]) : 0.0f);
        }
        __syncthreads();
        // squared norms of the seeds (warp w takes centroids w, w+4, ...; lanes
        // split the dimensions); later rounds get them from the update
        for (int j = warp; j < CP; j += 4) {
            float s2 = 0.0f;
#pragma unroll
            for (int x = lane; x < D; x += 32) s2 = fmaf(cent[j * D + x], cent[j * D + x], s2);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
            if (lane == 0) {
                cnp_s[0][j] = s2;
                cnp_s[1][j] = cnp_s[2][j] = cnp_s[3][j] = 0.0f;
            }
        }
        __syncthreads();

        const int rounds = a.iters > 0 ? a.iters : 1;
        for (int it = 0; it < rounds; ++it) {
            // ---- assignment: q.c on tensor cores, argmin over centroids ----
            // warp w: rows 32w..32w+31 as two 16-row MMA tiles; per 16-dim step one
            // ldmatrix of each query tile and one of the centroids' hi and lo parts
            // (shared by both tiles)
            const int nt = (ce + 7) >> 3;  // 8-wide centroid tiles
            float bestd[2][2];
            int besti[2][2];
#pragma unroll
            for (int m = 0; m < 2; ++m)
#pragma unroll
                for (int h = 0; h < 2; ++h) { bestd[m][h] = __int_as_float(0x7f800000); besti[m][h] = 0; }
            // lane roles in the x4 loads: query row (l % 16) at column half l / 16;
            // centroid row (l % 8) of the hi (l < 16) or lo part at column half (l / 8) % 2
            const __nv_bfloat16 *qa = qs + (warp * 32 + (lane & 15)) * LDQ + (lane >> 4) * 8;
            for (int t = 0; t < nt; ++t) {
                const __nv_bfloat16 *cb = (lane < 16 ? chi : clo) + (t * 8 + (lane & 7)) * LDQ + ((lane >> 3) & 1) * 8;
                // eight independent accumulation chains: query tile m, centroid
                // part (hi, lo) and the parity of the 16-dimension step
                float acc[2][2][2][4];
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int kp = 0; kp < 2; ++kp)
#pragma unroll
                            for (int u = 0; u < 4; ++u) acc[m][h][kp][u] = 0.0f;
#pragma unroll
                for (int k0 = 0; k0 < D; k0 += 16) {
                    const int kp = (k0 >> 4) & 1;
                    uint32_t bf[4];  // hi (k0..7, k8..15), lo (k0..7, k8..15)
                    ldsm_x4(bf, cb + k0);
#pragma unroll
                    for (int m = 0; m < 2; ++m) {
                        uint32_t af[4];
                        ldsm_x4(af, qa + m * 16 * LDQ + k0);
                        mma_bf16_16816(acc[m][0][kp], af, bf[0], bf[1]);
                        mma_bf16_16816(acc[m][1][kp], af, bf[2], bf[3]);
                    }
                }
                float cn[2];  // squared norms of this lane's two centroids
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int j = t * 8 + 2 * cq + u;
                    cn[u] = (cnp_s[0][j] + cnp_s[1][j]) + (cnp_s[2][j] + cnp_s[3][j]);
                }
                // acc[m][.][.][0..1]: row g, centroids t*8+2cq+{0,1}; [2..3]: row g+8
#pragma unroll
                for (int m = 0; m < 2; ++m)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int j = t * 8 + 2 * cq + u;
                            const int e = 2 * h + u;
                            const float dot = (acc[m][0][0][e] + acc[m][0][1][e]) + (acc[m][1][0][e] + acc[m][1][1][e]);
                            const float dj = j < ce ? fmaf(-2.0f, dot, cn[u]) : __int_as_float(0x7f800000);
                            if (dj < bestd[m][h]) { bestd[m][h] = dj; besti[m][h] = j; }
                        }
            }
            // combine the four lanes of each row (ties to the lower index)
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int r0 = warp * 32 + m * 16;
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
            // ---- cluster sizes of this warp's 32 rows (ballots), before the barrier ----
            __syncwarp();
            {
                const int best = assign_s[tid];  // row tid belongs to this warp
                for (int j = 0; j < ce; ++j) {
                    const uint32_t m = __ballot_sync(0xffffffffu, best == j);
                    if (lane == 0) wcnt_s[warp][j] = __popc(m);
                }
            }
            __syncthreads();
            if (a.iters == 0) break;  // sizes from the seeds, no update

            // ---- update: sums = onehot^T (16 x 128) . Q (128 x D) ----
            // A rows are the clusters (up to 16: one MMA tile), A columns the
            // block's rows (1 where the row is assigned to the cluster); warp w
            // takes the column tiles of dimensions [w*D/4, (w+1)*D/4)
            {
                constexpr int NT = D / 32;  // 8-wide column tiles per warp
                float acc[2][NT][4];            // [parity of the 16-row step][column tile]
#pragma unroll
                for (int kp = 0; kp < 2; ++kp)
#pragma unroll
                    for (int t = 0; t < NT; ++t)
#pragma unroll
                        for (int u = 0; u < 4; ++u) acc[kp][t][u] = 0.0f;
                const int n0w = warp * NT * 8;
#pragma unroll
                for (int k0 = 0; k0 < 128; k0 += 16) {
                    const int kp = (k0 >> 4) & 1;
                    const int q0 = assign_s[k0 + 2 * cq], q1 = assign_s[k0 + 2 * cq + 1];
                    const int q8 = assign_s[k0 + 2 * cq + 8], q9 = assign_s[k0 + 2 * cq + 9];
                    uint32_t af[4];
                    af[0] = onehot_pair(q0 == g, q1 == g);
                    af[1] = onehot_pair(q0 == g + 8, q1 == g + 8);
                    af[2] = onehot_pair(q8 == g, q9 == g);
                    af[3] = onehot_pair(q8 == g + 8, q9 == g + 8);
#pragma unroll
                    for (int t = 0; t < NT; t += 2) {
                        // matrices: rows k0..k0+7 / k0+8..k0+15 of column tiles t, t+1
                        const int mi = lane >> 3;
                        const __nv_bfloat16 *ra =
                            qs + (k0 + (mi & 1) * 8 + (lane & 7)) * LDQ + n0w + (t + (mi >> 1)) * 8;
                        uint32_t b[4];
                        ldsm_x4_trans(b, ra);
                        mma_bf16_16816(acc[kp][t], af, b[0], b[1]);
                        mma_bf16_16816(acc[kp][t + 1], af, b[2], b[3]);
                    }
                }
                // acc[.][t]: [0..1] cluster g, dimensions n0w+8t+2cq+{0,1}; [2..3] cluster g+8.
                // Each updated centroid also leaves the squared norm of this warp's
                // D/4 dimensions of it for the next assignment (the four lanes of a
                // quad hold one cluster's values)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int j = g + 8 * h;
                    const int c = j < ce ? wcnt_s[0][j] + wcnt_s[1][j] + wcnt_s[2][j] + wcnt_s[3][j] : 0;
                    // c == 0: an empty cluster keeps its centroid (and its norm)
                    const float inv = c > 0 ? __frcp_rn((float)c) : 0.0f;  // sum / size as sum * (1/size)
                    float pn = 0.0f;
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        const int x = n0w + 8 * t + 2 * cq;
                        const float c0 = __fmul_rn(acc[0][t][2 * h] + acc[1][t][2 * h], inv);
                        const float c1 = __fmul_rn(acc[0][t][2 * h + 1] + acc[1][t][2 * h + 1], inv);
                        pn = fmaf(c0, c0, pn);
                        pn = fmaf(c1, c1, pn);
                        if (c > 0) {
                            put(j, x, c0);
                            put(j, x + 1, c1);
                        }
                    }
                    pn += __shfl_xor_sync(0xffffffffu, pn, 1);
                    pn += __shfl_xor_sync(0xffffffffu, pn, 2);
                    if (c > 0 && cq == 0) cnp_s[warp][j] = pn;
                }
            }
            __syncthreads();
        }

        // ---- outputs ----
        const float mul = a.logit_mul;  // scale * log2(e)
        for (int e = tid; e < C * D; e += kKmThreads) {
            const int j = e / D, x = e % D;
            const float c = j < ce ? cent[j * D + x] : 0.0f;
            const int64_t o = (row * C + j) * (int64_t)D + x;
            a.cent16[o] = __float2half_rn(c * mul);
            if (a.cent_out) a.cent_out[o] = c;
        }
        if (tid < C) {
            const int c = tid < ce ? wcnt_s[0][tid] + wcnt_s[1][tid] + wcnt_s[2][tid] + wcnt_s[3][tid] : 0;
            a.weight[row * C + tid] = (float)c / (float)n;
            if (a.sizes_out) a.sizes_out[row * C + tid] = c;
        }
        __syncthreads();
    }
}

}  // namespace

size_t kmeans_smem_bytes(int D, int C) {
    const int ldq = D + 8, cp = C <= 8 ? 8 : 16;
    return (size_t)128 * ldq * 2 + sizeof(float) * cp * D + 2 * (size_t)cp * ldq * 2;
}

template <int D>
cudaError_t launch_kmeans_d(const KmeansArgs &a, int num_sms, cudaStream_t stream) {
    const size_t smem = kmeans_smem_bytes(D, a.C);
    cudaError_t e = cudaFuncSetAttribute(kmeans_qblock_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kmeans_qblock_kernel<D>, kKmThreads,
                                                      smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    int64_t grid = a.rows;
    const int64_t cap = (int64_t)num_sms * per_sm;  // every CTA resident: an even share each
    if (grid > cap) grid = cap;
    kmeans_qblock_kernel<D><<<(unsigned)grid, kKmThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_kmeans(const KmeansArgs &a, int num_sms, cudaStream_t stream) {
    if (a.rows < 1) return cudaSuccess;
    return a.D == 128 ? launch_kmeans_d<128>(a, num_sms, stream)
                      : launch_kmeans_d<64>(a, num_sms, stream);
}

}  // namespace abatt
