// kernels.cuh -- argument blocks and launchers of the abatt kernels.
#pragma once

#include "common.cuh"

namespace abatt {

// Element strides of Q, K, V, O: element (beta, h, t, x) sits at
// beta*sB + h*sH + t*sT + x.  [B][H][N][d]: sT = d, sH = N*d, sB = H*N*d;
// [B][N][H][d]: sT = H*d, sH = d, sB = N*H*d.
struct Strides {
    int64_t sT, sH, sB;
    int H;
    // bh = beta*H + h < 2^16 (B*H <= 65535 is a limit of the ABI): 32-bit division
    __host__ __device__ int64_t head_base(int64_t bh) const {
        const int b = (int)bh / H;
        return b * sB + ((int)bh - b * H) * sH;
    }
};

// ---- IBCS part 1: per-query-block k-means ---------------------------------
struct KmeansArgs {
    const __nv_bfloat16 *Q;  // strided as st
    Strides st;
    int64_t rows;            // B*H*nQ
    int nQ, N, D, C, iters;
    float logit_mul;         // scale * log2(e), folded into the GEMM operand
    __half *cent16;          // [rows*C][D] scoring operand: fp16 of the scaled centroids
    float *weight;           // [rows][C]  n_j / n
    float *cent_out;         // optional [rows][C][D]
    int32_t *sizes_out;      // optional [rows][C]
};
size_t kmeans_smem_bytes(int D, int C);
cudaError_t launch_kmeans(const KmeansArgs &a, int num_sms, cudaStream_t stream);

// ---- IBCS part 2: centroid . key softmax mass per key block -----------------
// For every centroid row (head hd, local row m < MC = nQ*C) and every 128-key
// tile T: base-2 logits x = c'.k (c' pre-scaled), running max and sum, and
// per key block b of the tile the partial mass r = sum_{t in b} 2^(x - mref_T)
// where mref_T is the row's running maximum after tile T.
struct ScoreArgs {
    int heads;     // B*H
    int N, D, Bk;
    int MC;        // centroid rows per head (nQ*C)
    int nT;        // key tiles per head, ceil(N/128)
    int ldr;       // row stride of r in floats (nT * 128/Bk)
    int nchunk;    // the key tiles are split into nchunk ranges of chunk_tiles (one CTA each)
    float last_weight;  // coarse scoring (Bk == 1): weight of the last key column (n_last / Bk)
    int chunk_tiles;
    // coarse scoring (Bk == 1) only:
    //   mode 0: block values to r (+ mref), combined by launch_combine_cols;
    //   mode 1: each centroid row's (max, sum) to mz only;
    //   mode 2: p directly, from the merged (max, sum) of a mode-1 pass over the
    //           same grid -- the C centroid rows of a query block are C adjacent
    //           lanes of one warp, so C must divide 32
    int mode;
    int C;
    const float *weight;  // [heads*MC] n_j / n (mode 2)
    float *p;             // [heads*MC/C][N] (mode 2)
    float *r;      // [heads*MC][ldr]
    float *mref;   // [heads*MC][nT], running maximum within the tile's chunk
    float2 *mz;    // [heads*MC][nchunk] (max, sum) of each chunk in base 2
    WsHeader *hdr;
    uint64_t wait_ns;
    int stall;     // test hook: the copy producer stops after its first tile
};
struct ScoreMaps {
    CUtensorMap a;  // fp16 scaled centroids [heads][MC][D], box (64, 128, 1)
    CUtensorMap k;  // fp16 keys [heads][N][D], box (64, 128, 1)
};
cudaError_t launch_score(const ScoreArgs &a, const ScoreMaps &maps, int num_sms,
                         cudaStream_t stream);

// Keys to fp16 for the scoring GEMM (bf16 -> fp16 is exact inside fp16's
// normal range; magnitudes beyond 65504 saturate).  n8 = elements / 8.
cudaError_t launch_keys_f16(const __nv_bfloat16 *K, __half *K16, int64_t n8, int num_sms,
                            cudaStream_t stream);
// Same from strided keys: K16[bh][t] = K at (bh, t), heads*N rows of D.
cudaError_t launch_keys_f16_strided(const __nv_bfloat16 *K, const Strides &st, __half *K16, int64_t heads,
                                    int N, int D, int num_sms, cudaStream_t stream);

// Mean key of every key block, to fp16 (coarse scoring): Kbar[head][b] =
// mean of the block's valid keys.
cudaError_t launch_keys_block_mean(const __nv_bfloat16 *K, const Strides &st, __half *Kbar, int64_t heads,
                                   int N, int D, int Bk, int nK, int num_sms, cudaStream_t stream);

// Combine the C centroids of each query block into p (see score.cu).
struct CombineArgs {
    int64_t rows;  // query blocks
    int C, nK, nT, ldr, Bk, nchunk;
    const float *r, *mref, *weight;
    const float2 *mz;
    float *p;      // [rows][nK]
};
cudaError_t launch_combine(const CombineArgs &a, int num_sms, cudaStream_t stream);
// Same for coarse scoring: r holds one value per key block, tiles of 128 blocks.
cudaError_t launch_combine_cols(const CombineArgs &a, int num_sms, cudaStream_t stream);

// ---- SIP sampler --------------------------------------------------------
struct SampleArgs {
    const float *p;  // [rows][nK]
    int64_t rows;
    int nK, nK_pad, nQ, H;
    int64_t M;
    uint32_t b_off, h_off;  // global index of the first batch element / head (Philox counter)
    int topk;               // 1: keep the M largest estimates (weight 1) instead of drawing
    int paired;             // 1: Philox counter word 1 is i/2 (query blocks 2j, 2j+1 share draws)
    uint32_t key0, key1;
    int capacity;
    int32_t *counts, *idx;
    float *logw;
    uint32_t *status;
};
size_t sample_smem_bytes(int nK);
cudaError_t launch_sample(const SampleArgs &a, int num_sms, cudaStream_t stream);

// ---- gather attention -----------------------------------------------------
// Query blocks are processed in pairs of neighbours of the same head: pair
// (h, j) holds blocks 2j and 2j+1 of head h (the last pair of a head is a
// single block when nQ is odd).  A pre-pass lays the pair's two lists out as
// one array of three ascending segments, [blocks both rows drew | row 0 only
// | row 1 only] (nb, na, nc entries).  Row 0 walks [both | row 0 only], row 1
// walks [both | row 1 only]: each row runs over exactly its own blocks, and
// the 128-key tiles that lie wholly inside the shared segment are gathered
// once for both rows.
__host__ __device__ __forceinline__ int64_t pairs_per_head(int nQ) { return (nQ + 1) / 2; }

// Rows of pair `pr`: first row, and the second row or -1.
__host__ __device__ __forceinline__ void pair_rows(int64_t pr, int nQ, int64_t *r0, int64_t *r1) {
    const int64_t pph = pairs_per_head(nQ);
    const int64_t h = pr / pph, j = pr - h * pph;
    *r0 = h * nQ + 2 * j;
    *r1 = (2 * j + 1 < nQ) ? *r0 + 1 : -1;
}

struct PairArgs {
    int64_t rows, pairs;
    int nQ, nK, capacity, cap_u;
    int ragged;     // N % Bk != 0: the last key block is partial
    int bpt;        // key blocks per 128-key tile
    int cap_w;      // row stride of ulw (nK rounded up to 8)
    const int32_t *counts, *idx;
    const float *logw;
    int32_t *useg;  // [pairs][4]       nb, na, nc (segment lengths), position of a partial last block (-1: none)
    int32_t *ublk;  // [pairs][cap_u]   [both | row 0 only | row 1 only], ascending within each
    float *ulw;     // [pairs][2][cap_w] row s's log-weights in base 2 (log2(e) * -ln pi) in the order of its
                    // sequence ([both | own]), -inf up to its last tile's end
    uint32_t *status;
};
cudaError_t launch_pair_union(const PairArgs &a, int num_sms, cudaStream_t stream);

struct AttnArgs {
    int64_t rows, pairs;  // query blocks, row pairs
    int nQ, N, D, Bk, nK;
    int cap_u, cap_w;
    int k_fold;        // K tiles as boxes of 8-row groups (needs N % 8 == 0)
    int kf_gb, kf_zb;  // k_fold: group coordinate b*kf_gb + blk*Bk/8, outer coordinate b*kf_zb + h
    Strides st;        // of O (and of Q, K, V in the maps)
    float scale_log2;  // scale * log2(e)
    const int32_t *useg, *ublk;
    const float *ulw;
    __nv_bfloat16 *O;  // strided as st
    float *lse;        // optional [B*H][N]
    WsHeader *hdr;
    uint64_t wait_ns;
    int stall;         // test hook: the copy producer stops after its first K/V tile pair
};
struct AttnMaps {
    CUtensorMap q;  // (D, N, H, B), box (64, 128, 1, 1)
    CUtensorMap k;  // k_fold: (64, 8 rows, D/64 chunks, groups, outer), box (64, 8, D/64, Bk/8, 1)
                    // else:   (D, N, H, B), box (64, Bk, 1, 1)
    CUtensorMap v;  // (64, N rows, D/64 chunks, H, B), box (64, Bk, D/64, 1, 1)
};
cudaError_t launch_attention(const AttnArgs &a, const AttnMaps &maps, int num_sms,
                             cudaStream_t stream);

}  // namespace abatt
