// abatt.cu -- host side of the C ABI declared in include/abatt.h: argument
// validation, workspace layout, TMA descriptor encoding and the launch
// sequence of each call.  No allocation, no synchronisation except in
// abatt_read_status.
#include <math.h>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <string.h>

#include "kernels.cuh"

using namespace abatt;

namespace {

constexpr uint64_t kWaitNs = 500000000ull;  // bounded waits give up after ~0.5 s

// Test hooks (abatt_test_set): the bounded-wait limit and the producer stall.
std::atomic<uint64_t> g_wait_ns{kWaitNs};
std::atomic<uint32_t> g_stall{0};
constexpr float kLog2eF = 1.4426950408889634f;

struct Geom {
    int B, H, N, d, Bq, Bk, C, I, nQ, nK, nT, ldr;
    int nTc;  // coarse scoring: tiles of 128 key blocks; r rows then hold nTc*128 values
    int64_t rows, heads, M;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

Strides strides_of(const Geom &g, const abatt_config *cfg) {
    Strides s;
    s.H = g.H;
    if (cfg->layout == ABATT_LAYOUT_BNHD) {
        s.sT = (int64_t)g.H * g.d;
        s.sH = g.d;
    } else {
        s.sT = g.d;
        s.sH = (int64_t)g.N * g.d;
    }
    s.sB = (int64_t)g.H * g.N * g.d;
    return s;
}

// The scoring kernel runs one CTA per (centroid tile, head, key-range chunk),
// one CTA per SM at a time.  Split the key tiles into the fewest chunks (at
// most kMaxScoreChunks, each of at least 24 tiles) whose CTA count fills its
// last wave of SMs to 95 %, else take the best fill found.
constexpr int kMaxScoreChunks = 8;
void score_chunks(int nT, int64_t ctas, int sms, int *nchunk, int *chunk_tiles) {
    const int nmax = nT / 24 < 1 ? 1 : (nT / 24 > kMaxScoreChunks ? kMaxScoreChunks : nT / 24);
    int best = 1;
    double best_fill = 0.0;
    for (int n = 1; n <= nmax; ++n) {
        const int per = (nT + n - 1) / n;
        const int neff = (nT + per - 1) / per;  // no empty chunk
        const double waves = (double)(ctas * neff) / (sms > 0 ? sms : 1);
        const double fill = waves / ceil(waves);
        if (fill > best_fill + 1e-9) {
            best_fill = fill;
            best = n;
        }
        if (fill >= 0.95) break;
    }
    *chunk_tiles = (nT + best - 1) / best;
    *nchunk = (nT + *chunk_tiles - 1) / *chunk_tiles;
}

abatt_status validate(const abatt_shape *s, const abatt_config *c, Geom *g) {
    if (!s || !c) return ABATT_ERR_INVALID_ARG;
    if (s->B <= 0 || s->H <= 0 || s->N <= 0 || s->d <= 0) return ABATT_ERR_INVALID_ARG;
    if (c->budget_bp < 0 || !(c->scale > 0.0f) || !isfinite(c->scale)) return ABATT_ERR_INVALID_ARG;
    if (c->batch_offset < 0 || c->head_offset < 0) return ABATT_ERR_INVALID_ARG;
    if (c->selection != ABATT_SELECT_SIP && c->selection != ABATT_SELECT_TOPK) return ABATT_ERR_INVALID_ARG;
    if (c->scoring != ABATT_SCORE_KEYS && c->scoring != ABATT_SCORE_BLOCK_MEANS) return ABATT_ERR_INVALID_ARG;
    if (c->layout != ABATT_LAYOUT_BHND && c->layout != ABATT_LAYOUT_BNHD) return ABATT_ERR_INVALID_ARG;
    if (c->draws != ABATT_DRAWS_INDEPENDENT && c->draws != ABATT_DRAWS_PAIRED) return ABATT_ERR_INVALID_ARG;
    if (s->d != 64 && s->d != 128) return ABATT_ERR_UNSUPPORTED;
    if (c->q_block != 128) return ABATT_ERR_UNSUPPORTED;
    if (c->kv_block != 16 && c->kv_block != 32 && c->kv_block != 64 && c->kv_block != 128)
        return ABATT_ERR_UNSUPPORTED;
    if (c->clusters < 1 || c->clusters > 16) return ABATT_ERR_UNSUPPORTED;
    if (c->kmeans_iters < 0 || c->kmeans_iters > 64) return ABATT_ERR_UNSUPPORTED;
    g->B = s->B; g->H = s->H; g->N = s->N; g->d = s->d;
    g->Bq = c->q_block; g->Bk = c->kv_block; g->C = c->clusters; g->I = c->kmeans_iters;
    g->nQ = (s->N + 127) / 128;
    g->nK = (s->N + g->Bk - 1) / g->Bk;
    g->nT = (s->N + 127) / 128;
    g->ldr = g->nT * (128 / g->Bk);
    g->nTc = (g->nK + 127) / 128;
    g->heads = (int64_t)s->B * s->H;
    g->rows = g->heads * g->nQ;
    if (g->nK > 32767) return ABATT_ERR_UNSUPPORTED;
    if (g->rows >= (int64_t(1) << 31) || g->heads > 65535) return ABATT_ERR_UNSUPPORTED;
    if ((int64_t)s->N * s->d * g->heads >= (int64_t(1) << 40)) return ABATT_ERR_UNSUPPORTED;
    g->M = ((int64_t)c->budget_bp * g->nK + 5000) / 10000;
    if (c->selection == ABATT_SELECT_TOPK && g->nK > 10240) return ABATT_ERR_UNSUPPORTED;
    return ABATT_OK;
}

// ---- workspace layout ----------------------------------------------------------
struct Layout {
    size_t hdr, cent16, k16, weight, r, mref, mz;  // select
    size_t useg, ublk, ulw;                               // attention (pair segments)
    size_t p, counts, idx, logw;                          // forward
    size_t total;
};

int64_t pairs_of(const Geom &g) { return g.heads * pairs_per_head(g.nQ); }

Layout layout(abatt_call call, const Geom &g) {
    Layout L;
    memset(&L, 0, sizeof L);
    size_t off = 0;
    L.hdr = off;
    off += sizeof(WsHeader);
    if (call == ABATT_CALL_SELECT || call == ABATT_CALL_FORWARD) {
        const size_t crow = (size_t)g.rows * g.C;
        L.cent16 = off;  off = align256(off + crow * g.d * 2);
        L.k16 = off;     off = align256(off + (size_t)g.heads * g.N * g.d * 2);
        L.weight = off;  off = align256(off + crow * 4);
        const size_t ldr = std::max((size_t)g.ldr, (size_t)g.nTc * 128);  // either scoring rule
        L.r = off;       off = align256(off + crow * ldr * 4);
        L.mref = off;    off = align256(off + crow * std::max(g.nT, g.nTc) * 4);
        L.mz = off;      off = align256(off + crow * 8 * kMaxScoreChunks);
    }
    if (call == ABATT_CALL_ATTENTION || call == ABATT_CALL_FORWARD) {
        const size_t pairs = (size_t)pairs_of(g);
        L.useg = off; off = align256(off + pairs * 16);
        L.ublk = off; off = align256(off + pairs * g.nK * 4);
        L.ulw = off;  off = align256(off + pairs * 2 * (size_t)((g.nK + 7) & ~7) * 4);
    }
    if (call == ABATT_CALL_FORWARD) {
        L.p = off;      off = align256(off + (size_t)g.rows * g.nK * 4);
        L.counts = off; off = align256(off + (size_t)g.rows * 4);
        L.idx = off;    off = align256(off + (size_t)g.rows * g.nK * 4);
        L.logw = off;   off = align256(off + (size_t)g.rows * g.nK * 4);
    }
    L.total = off;
    return L;
}

// ---- per-device cache --------------------------------------------------------
std::mutex g_mu;
int g_sms[64];

abatt_status device_sms(int *sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ABATT_ERR_CUDA;
    if (dev < 0 || dev >= 64) return ABATT_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return ABATT_ERR_CUDA;
        g_sms[dev] = n;
    }
    *sms = g_sms[dev];
    return ABATT_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D map of 16-bit elements (bf16 unless stated) over [outer][rows][d] with
// a (64, box_rows, 1) box, 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap *m, const void *base, int d, int64_t rows, int64_t outer, int box_rows,
              CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)outer};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, dtype, 3, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 map of `rank` dimensions (dims[0] innermost, strides in bytes of
// dims 1..rank-1) with 128-byte swizzle and a 64-element inner box.
bool make_map_nd(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
                 const cuuint64_t *strides, const cuuint32_t *box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename T>
T *at(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

abatt_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ABATT_OK : ABATT_ERR_CUDA; }

abatt_status check_ws(abatt_call call, const Geom &g, void *ws, size_t bytes) {
    if (!ws) return ABATT_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return ABATT_ERR_ALIGNMENT;
    if (bytes < layout(call, g).total) return ABATT_ERR_WORKSPACE;
    return ABATT_OK;
}

// ---- the three stages ------------------------------------------------------
abatt_status run_select(const void *Q, const void *K, const Geom &g, const abatt_config *cfg,
                        float *p, float *cent_out, int32_t *sizes_out, void *ws, const Layout &L,
                        int sms, cudaStream_t st) {
    KmeansArgs ka;
    ka.Q = static_cast<const __nv_bfloat16 *>(Q);
    ka.st = strides_of(g, cfg);
    ka.rows = g.rows; ka.nQ = g.nQ; ka.N = g.N; ka.D = g.d; ka.C = g.C; ka.iters = g.I;
    ka.logit_mul = cfg->scale * kLog2eF;
    ka.cent16 = at<__half>(ws, L.cent16);
    ka.weight = at<float>(ws, L.weight);
    ka.cent_out = cent_out;
    ka.sizes_out = sizes_out;
    cudaError_t e = launch_kmeans(ka, sms, st);
    if (e != cudaSuccess) return ABATT_ERR_CUDA;

    __half *k16 = at<__half>(ws, L.k16);
    const bool coarse = cfg->scoring == ABATT_SCORE_BLOCK_MEANS;
    // the scoring GEMM's key operand: fp16 keys, or fp16 block-mean keys
    const __nv_bfloat16 *Kb = static_cast<const __nv_bfloat16 *>(K);
    if (coarse)
        e = launch_keys_block_mean(Kb, ka.st, k16, g.heads, g.N, g.d, g.Bk, g.nK, sms, st);
    else if (cfg->layout == ABATT_LAYOUT_BHND)
        e = launch_keys_f16(Kb, k16, g.heads * g.N * g.d / 8, sms, st);
    else
        e = launch_keys_f16_strided(Kb, ka.st, k16, g.heads, g.N, g.d, sms, st);
    if (e != cudaSuccess) return ABATT_ERR_CUDA;

    ScoreMaps sm;
    const int64_t MC = (int64_t)g.nQ * g.C;
    const int nkeys = coarse ? g.nK : g.N;  // rows of the key operand per head
    if (!make_map(&sm.a, ka.cent16, g.d, MC, g.heads, 128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !make_map(&sm.k, k16, g.d, nkeys, g.heads, 128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
        return ABATT_ERR_CUDA;
    ScoreArgs sa;
    sa.heads = (int)g.heads; sa.N = nkeys; sa.D = g.d; sa.Bk = coarse ? 1 : g.Bk; sa.MC = (int)MC;
    sa.nT = coarse ? g.nTc : g.nT;
    sa.ldr = coarse ? g.nTc * 128 : g.ldr;
    // coarse: the last block's share is weighted by its valid keys over a full block
    sa.last_weight = coarse ? (float)(g.N - (g.nK - 1) * g.Bk) / (float)g.Bk : 1.0f;
    score_chunks(sa.nT, ((int)MC + 127) / 128 * g.heads, sms, &sa.nchunk, &sa.chunk_tiles);
    sa.r = at<float>(ws, L.r);
    sa.mref = at<float>(ws, L.mref);
    sa.mz = at<float2>(ws, L.mz);
    sa.hdr = at<WsHeader>(ws, L.hdr);
    sa.wait_ns = g_wait_ns.load();
    sa.stall = (g_stall.load() & ABATT_TEST_STALL_SCORE) ? 1 : 0;
    sa.C = g.C;
    sa.weight = ka.weight;
    sa.p = p;
    sa.mode = 0;
    if (coarse && 32 % g.C == 0) {
        // two passes over the (cheap) block-mean GEMM: the centroids' softmax
        // statistics, then p summed over each query block's centroid lanes
        sa.mode = 1;
        if ((e = launch_score(sa, sm, sms, st)) != cudaSuccess) return ABATT_ERR_CUDA;
        sa.mode = 2;
        return cuda_status(launch_score(sa, sm, sms, st));
    }
    e = launch_score(sa, sm, sms, st);
    if (e != cudaSuccess) return ABATT_ERR_CUDA;

    CombineArgs ca;
    ca.rows = g.rows; ca.C = g.C; ca.nK = g.nK; ca.nT = sa.nT; ca.ldr = sa.ldr; ca.Bk = g.Bk;
    ca.r = sa.r; ca.mref = sa.mref; ca.weight = ka.weight; ca.mz = sa.mz; ca.p = p;
    ca.nchunk = sa.nchunk;
    return cuda_status(coarse ? launch_combine_cols(ca, sms, st) : launch_combine(ca, sms, st));
}

abatt_status run_sample(const float *p, const Geom &g, const abatt_config *cfg, int32_t *counts,
                        int32_t *idx, float *logw, int capacity, WsHeader *hdr, int sms,
                        cudaStream_t st) {
    SampleArgs a;
    a.p = p; a.rows = g.rows; a.nK = g.nK; a.nK_pad = (g.nK + 3) & ~3; a.nQ = g.nQ; a.H = g.H;
    a.M = g.M;
    a.topk = cfg->selection == ABATT_SELECT_TOPK ? 1 : 0;
    a.paired = cfg->draws == ABATT_DRAWS_PAIRED ? 1 : 0;
    a.b_off = (uint32_t)cfg->batch_offset;
    a.h_off = (uint32_t)cfg->head_offset;
    a.key0 = (uint32_t)(cfg->seed & 0xffffffffu);
    a.key1 = (uint32_t)(cfg->seed >> 32);
    a.capacity = capacity; a.counts = counts; a.idx = idx; a.logw = logw;
    a.status = &hdr->status;
    return cuda_status(launch_sample(a, sms, st));
}

PairArgs pair_args(const Geom &g, const int32_t *counts, const int32_t *idx, const float *logw, int capacity,
                   void *ws, const Layout &L) {
    PairArgs pa;
    pa.rows = g.rows; pa.pairs = pairs_of(g); pa.nQ = g.nQ; pa.nK = g.nK; pa.capacity = capacity; pa.cap_u = g.nK;
    pa.counts = counts; pa.idx = idx; pa.logw = logw;
    pa.ragged = (g.N % g.Bk) != 0 ? 1 : 0;
    pa.bpt = 128 / g.Bk;
    pa.cap_w = (g.nK + 7) & ~7;
    pa.useg = at<int32_t>(ws, L.useg);
    pa.ublk = at<int32_t>(ws, L.ublk);
    pa.ulw = at<float>(ws, L.ulw);
    pa.status = &at<WsHeader>(ws, L.hdr)->status;
    return pa;
}

// Pair segments of every pair of query blocks (the first launch of attention).
abatt_status run_plan(const Geom &g, const int32_t *counts, const int32_t *idx, const float *logw,
                      int capacity, void *ws, const Layout &L, int sms, cudaStream_t st) {
    const PairArgs pa = pair_args(g, counts, idx, logw, capacity, ws, L);
    return cuda_status(launch_pair_union(pa, sms, st));
}

// Gather attention from the pair segments in the workspace (the second launch).
abatt_status run_planned(const void *Q, const void *K, const void *V, const Geom &g,
                         const abatt_config *cfg, void *O, float *lse, void *ws, const Layout &L, int sms,
                         cudaStream_t st) {
    const PairArgs pa = pair_args(g, nullptr, nullptr, nullptr, 1, ws, L);
    const int CH = g.d / 64;
    const Strides sd = strides_of(g, cfg);
    const bool bnhd = cfg->layout == ABATT_LAYOUT_BNHD;
    // K as boxes of 8-row groups: the batch index folds into the group index
    // ([B][N][H][d]: sB = N*sT) or into the outer index ([B][H][N][d]: sB = H*sH)
    const int64_t groups = bnhd ? (int64_t)g.B * (g.N / 8) : g.N / 8;
    const int64_t outer = bnhd ? g.H : g.heads;
    const bool fold = (g.N % 8) == 0 && groups < (int64_t(1) << 31) && outer < (int64_t(1) << 31);
    const cuuint64_t sT2 = (cuuint64_t)sd.sT * 2, sH2 = (cuuint64_t)sd.sH * 2, sB2 = (cuuint64_t)sd.sB * 2;
    AttnMaps m;
    {
        const cuuint64_t dims[4] = {(cuuint64_t)g.d, (cuuint64_t)g.N, (cuuint64_t)g.H, (cuuint64_t)g.B};
        const cuuint64_t strides[3] = {sT2, sH2, sB2};
        const cuuint32_t box[4] = {64, 128, 1, 1};
        if (!make_map_nd(&m.q, Q, 4, dims, strides, box)) return ABATT_ERR_CUDA;
    }
    if (fold) {
        const cuuint64_t dims[5] = {64, 8, (cuuint64_t)CH, (cuuint64_t)groups, (cuuint64_t)outer};
        const cuuint64_t strides[4] = {sT2, 128, 8 * sT2, sH2};
        const cuuint32_t box[5] = {64, 8, (cuuint32_t)CH, (cuuint32_t)(g.Bk / 8), 1};
        if (!make_map_nd(&m.k, K, 5, dims, strides, box)) return ABATT_ERR_CUDA;
    } else {
        const cuuint64_t dims[4] = {(cuuint64_t)g.d, (cuuint64_t)g.N, (cuuint64_t)g.H, (cuuint64_t)g.B};
        const cuuint64_t strides[3] = {sT2, sH2, sB2};
        const cuuint32_t box[4] = {64, (cuuint32_t)g.Bk, 1, 1};
        if (!make_map_nd(&m.k, K, 4, dims, strides, box)) return ABATT_ERR_CUDA;
    }
    {
        const cuuint64_t dims[5] = {64, (cuuint64_t)g.N, (cuuint64_t)CH, (cuuint64_t)g.H, (cuuint64_t)g.B};
        const cuuint64_t strides[4] = {sT2, 128, sH2, sB2};
        const cuuint32_t box[5] = {64, (cuuint32_t)g.Bk, (cuuint32_t)CH, 1, 1};
        if (!make_map_nd(&m.v, V, 5, dims, strides, box)) return ABATT_ERR_CUDA;
    }
    AttnArgs a;
    a.rows = g.rows; a.pairs = pairs_of(g); a.nQ = g.nQ; a.N = g.N; a.D = g.d; a.Bk = g.Bk;
    a.nK = g.nK; a.cap_u = g.nK; a.cap_w = pa.cap_w; a.k_fold = fold ? 1 : 0;
    a.kf_gb = bnhd ? g.N / 8 : 0;
    a.kf_zb = bnhd ? 0 : g.H;
    a.st = sd;
    a.scale_log2 = cfg->scale * kLog2eF;
    a.useg = pa.useg; a.ublk = pa.ublk; a.ulw = pa.ulw;
    a.O = static_cast<__nv_bfloat16 *>(O);
    a.lse = lse;
    a.hdr = at<WsHeader>(ws, L.hdr);
    a.wait_ns = g_wait_ns.load();
    a.stall = (g_stall.load() & ABATT_TEST_STALL_ATTENTION) ? 1 : 0;
    return cuda_status(launch_attention(a, m, sms, st));
}

abatt_status run_attention(const void *Q, const void *K, const void *V, const Geom &g,
                           const abatt_config *cfg, const int32_t *counts, const int32_t *idx,
                           const float *logw, int capacity, void *O, float *lse, void *ws,
                           const Layout &L, int sms, cudaStream_t st) {
    abatt_status s = run_plan(g, counts, idx, logw, capacity, ws, L, sms, st);
    if (s != ABATT_OK) return s;
    return run_planned(Q, K, V, g, cfg, O, lse, ws, L, sms, st);
}

// Scratch of abatt_attention_noalloc: status word and pair unions, in the
// library's device image (no allocation at call time).  Device code could
// name it directly; host code needs its address from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ABATT_NOALLOC_SCRATCH_BYTES];

// The address is only valid in the CUDA context it was looked up in (a reset
// device or a context a host made with the driver API loads the module
// again), so the cache is keyed on the current context's unique id.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

template <typename F>
F driver_fn(const char *name) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<F>(p);
}

// Unique id of the current context (0 and false when there is none).
bool current_ctx_id(unsigned long long *id) {
    static CtxGetCurrentFn get_cur = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        get_cur = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
        get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    });
    *id = 0;
    CUcontext ctx = nullptr;
    if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

struct ScratchEntry {
    unsigned long long ctx_id;  // context the address belongs to
    void *ptr;
};
std::mutex g_noalloc_mu;
ScratchEntry g_noalloc[64];  // per device: the last context seen there

// Device address of the scratch array in the current context, looked up with
// cudaGetSymbolAddress the first time a context calls.
abatt_status noalloc_scratch(void **ptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ABATT_ERR_CUDA;
    unsigned long long id = 0;
    const bool have_ctx = current_ctx_id(&id);
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!have_ctx || g_noalloc[dev].ctx_id != id || !g_noalloc[dev].ptr) {
        // with no context current, this makes the device's primary context current
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ABATT_ERR_CUDA;
        if (!current_ctx_id(&id)) return ABATT_ERR_CUDA;
        g_noalloc[dev].ctx_id = id;
        g_noalloc[dev].ptr = p;
    }
    *ptr = g_noalloc[dev].ptr;
    return ABATT_OK;
}

// 2^x through the FMA-pipe polynomial of the kernels (test hook).
template <int DEG>
__global__ void exp2_poly_kernel(const float *__restrict__ x, float *__restrict__ y, int64_t n) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x * 2;
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 2; i < n; i += stride) {
        const float2 v = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.0f);
        const float2 r = exp2_poly2<DEG>(v);
        y[i] = r.x;
        if (i + 1 < n) y[i + 1] = r.y;
    }
}

}  // namespace

extern "C" {

const char *abatt_version(void) { return "0.1.0"; }

const char *abatt_status_string(abatt_status s) {
    switch (s) {
        case ABATT_OK: return "ok";
        case ABATT_ERR_INVALID_ARG: return "invalid argument";
        case ABATT_ERR_UNSUPPORTED: return "unsupported shape or configuration";
        case ABATT_ERR_ALIGNMENT: return "misaligned pointer";
        case ABATT_ERR_WORKSPACE: return "workspace missing or too small";
        case ABATT_ERR_CUDA: return "CUDA runtime error";
        case ABATT_ERR_CAPACITY: return "a row drew more blocks than the list capacity";
        case ABATT_ERR_TIMEOUT: return "a bounded device wait ran out";
        case ABATT_ERR_DEVICE: return "device status word reports an error";
    }
    return "unknown status";
}

abatt_status abatt_workspace_size(abatt_call call, const abatt_shape *shape,
                                  const abatt_config *cfg, size_t *bytes) {
    if (!bytes) return ABATT_ERR_INVALID_ARG;
    if (call < ABATT_CALL_SELECT || call > ABATT_CALL_FORWARD) return ABATT_ERR_INVALID_ARG;
    Geom g;
    abatt_status s = validate(shape, cfg, &g);
    if (s != ABATT_OK) return s;
    *bytes = layout(call, g).total;
    return ABATT_OK;
}

abatt_status abatt_select(const void *Q, const void *K, const abatt_shape *shape,
                          const abatt_config *cfg, float *p, float *centroids,
                          int32_t *cluster_sizes, void *workspace, size_t workspace_bytes,
                          void *stream) {
    Geom g;
    abatt_status s = validate(shape, cfg, &g);
    if (s != ABATT_OK) return s;
    if (!Q || !K || !p) return ABATT_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(p)) return ABATT_ERR_ALIGNMENT;
    if ((s = check_ws(ABATT_CALL_SELECT, g, workspace, workspace_bytes)) != ABATT_OK) return s;
    int sms = 0;
    if ((s = device_sms(&sms)) != ABATT_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Layout L = layout(ABATT_CALL_SELECT, g);
    if (cudaMemsetAsync(workspace, 0, sizeof(WsHeader), st) != cudaSuccess) return ABATT_ERR_CUDA;
    return run_select(Q, K, g, cfg, p, centroids, cluster_sizes, workspace, L, sms, st);
}

abatt_status abatt_sample(const float *p, const abatt_shape *shape, const abatt_config *cfg,
                          int32_t *counts, int32_t *idx, float *logw, int capacity,
                          void *workspace, size_t workspace_bytes, void *stream) {
    Geom g;
    abatt_status s = validate(shape, cfg, &g);
    if (s != ABATT_OK) return s;
    if (!p || !counts || !idx || !logw || capacity < 1) return ABATT_ERR_INVALID_ARG;
    if ((s = check_ws(ABATT_CALL_SAMPLE, g, workspace, workspace_bytes)) != ABATT_OK) return s;
    int sms = 0;
    if ((s = device_sms(&sms)) != ABATT_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, sizeof(WsHeader), st) != cudaSuccess) return ABATT_ERR_CUDA;
    return run_sample(p, g, cfg, counts, idx, logw, capacity, static_cast<WsHeader *>(workspace),
                      sms, st);
}

abatt_status abatt_attention(const void *Q, const void *K, const void *V,
                             const abatt_shape *shape, const abatt_config *cfg,
                             const int32_t *counts, const int32_t *idx, const float *logw,
                             int capacity, void *O, float *lse, void *workspace,
                             size_t workspace_bytes, void *stream) {
    Geom g;
    abatt_status s = validate(shape, cfg, &g);
    if (s != ABATT_OK) return s;
    if (!Q || !K || !V || !O || !counts || !idx || !logw || capacity < 1)
        return ABATT_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
        return ABATT_ERR_ALIGNMENT;
    if ((s = check_ws(ABATT_CALL_ATTENTION, g, workspace, workspace_bytes)) != ABATT_OK) return s;
    int sms = 0;
    if ((s = device_sms(&sms)) != ABATT_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Layout L = layout(ABATT_CALL_ATTENTION, g);
    if (cudaMemsetAsync(workspace, 0, sizeof(WsHeader), st) != cudaSuccess) return ABATT_ERR_CUDA;
    return run_attention(Q, K, V, g, cfg, counts, idx, logw, capacity, O, lse, workspace, L, sms,
                         st);
}

abatt_status abatt_attention_plan(const abatt_shape *shape, const abatt_config *cfg,
                                  const int32_t *counts, const int32_t *idx, const float *logw,
                                  int capacity, void *workspace, size_t workspace_bytes,
                                  void *stream) {
    Geom g;
    abatt_status s = validate(shape, cfg, &g);
    if (s != ABATT_OK) return s;
    if (!counts || !idx || !logw || capacity < 1) return ABATT_ERR_INVALID_ARG;
    if ((s = check_ws(ABATT_CALL_ATTENTION, g, workspace, workspace_bytes)) != ABATT_OK) return s;
    int sms = 0;
    if ((s = device_sms(&sms)) != ABATT_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Layout L = layout(ABATT_CALL_ATTENTION, g);
    if (cudaMemsetAsync(workspace, 0, sizeof(WsHeader), st) != cudaSuccess) return ABATT_ERR_CUDA;
    return run_plan(g, counts, idx, logw, capacity, workspace, L, sms, st);
}

abatt_status abatt_attention_planned(const void *Q, const void *K, const void *V,
                                     const abatt_shape *shape, const abatt_config *cfg, void *O,
                                     float *lse, void *workspace, size_t workspace_bytes,
                                     void *stream) {
    Geom g;
    abatt_status s = validate(shape, cfg, &g);
    if (s != ABATT_OK) return s;
    if (!Q || !K || !V || !O) return ABATT_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return ABATT_ERR_ALIGNMENT;
    if ((s = check_ws(ABATT_CALL_ATTENTION, g, workspace, workspace_bytes)) != ABATT_OK) return s;
    int sms = 0;
    if ((s = device_sms(&sms)) != ABATT_OK) return s;
    const Layout L = layout(ABATT_CALL_ATTENTION, g);
    return run_planned(Q, K, V, g, cfg, O, lse, workspace, L, sms, static_cast<cudaStream_t>(stream));
}

abatt_status abatt_attention_noalloc(const void *Q, const void *K, const void *V,
                                     const abatt_shape *shape, const abatt_config *cfg,
                                     const int32_t *counts, const int32_t *idx, const float *logw,
                                     int capacity, void *O, float *lse, uint32_t *dev_status,
                                     void *stream) {
    Geom g;
    abatt_status s = validate(shape, cfg, &g);
    if (s != ABATT_OK) return s;
    if (!Q || !K || !V || !O || !counts || !idx || !logw || capacity < 1)
        return ABATT_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
        return ABATT_ERR_ALIGNMENT;
    const Layout L = layout(ABATT_CALL_ATTENTION, g);
    if (L.total > (size_t)ABATT_NOALLOC_SCRATCH_BYTES) return ABATT_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if ((s = noalloc_scratch(&scratch)) != ABATT_OK) return s;
    int sms = 0;
    if ((s = device_sms(&sms)) != ABATT_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // until this call's flags are copied there, dev_status reads "pending"
    if (dev_status && cudaMemsetAsync(dev_status, 0xFF, sizeof(uint32_t), st) != cudaSuccess)
        return ABATT_ERR_CUDA;
    // the status word must start at zero; the union lists are fully rewritten
    if (cudaMemsetAsync(scratch, 0, sizeof(WsHeader), st) != cudaSuccess) return ABATT_ERR_CUDA;
    s = run_attention(Q, K, V, g, cfg, counts, idx, logw, capacity, O, lse, scratch, L, sms, st);
    if (s != ABATT_OK) return s;
    if (dev_status && cudaMemcpyAsync(dev_status, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice,
                                      st) != cudaSuccess)
        return ABATT_ERR_CUDA;
    return ABATT_OK;
}

abatt_status abatt_forward(const void *Q, const void *K, const void *V,
                           const abatt_shape *shape, const abatt_config *cfg, void *O,
                           float *lse, void *workspace, size_t workspace_bytes, void *stream) {
    Geom g;
    abatt_status s = validate(shape, cfg, &g);
    if (s != ABATT_OK) return s;
    if (!Q || !K || !V || !O) return ABATT_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
        return ABATT_ERR_ALIGNMENT;
    if ((s = check_ws(ABATT_CALL_FORWARD, g, workspace, workspace_bytes)) != ABATT_OK) return s;
    int sms = 0;
    if ((s = device_sms(&sms)) != ABATT_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const Layout L = layout(ABATT_CALL_FORWARD, g);
    WsHeader *hdr = at<WsHeader>(workspace, L.hdr);
    if (cudaMemsetAsync(workspace, 0, sizeof(WsHeader), st) != cudaSuccess) return ABATT_ERR_CUDA;
    float *p = at<float>(workspace, L.p);
    int32_t *counts = at<int32_t>(workspace, L.counts);
    int32_t *idx = at<int32_t>(workspace, L.idx);
    float *logw = at<float>(workspace, L.logw);
    if ((s = run_select(Q, K, g, cfg, p, nullptr, nullptr, workspace, L, sms, st)) != ABATT_OK)
        return s;
    if ((s = run_sample(p, g, cfg, counts, idx, logw, g.nK, hdr, sms, st)) != ABATT_OK) return s;
    return run_attention(Q, K, V, g, cfg, counts, idx, logw, g.nK, O, lse, workspace, L, sms, st);
}

abatt_status abatt_forward_intermediates(void *workspace, const abatt_shape *shape,
                                         const abatt_config *cfg, float **p, int32_t **counts,
                                         int32_t **idx, float **logw) {
    Geom g;
    abatt_status s = validate(shape, cfg, &g);
    if (s != ABATT_OK) return s;
    if (!workspace) return ABATT_ERR_WORKSPACE;
    const Layout L = layout(ABATT_CALL_FORWARD, g);
    if (p) *p = at<float>(workspace, L.p);
    if (counts) *counts = at<int32_t>(workspace, L.counts);
    if (idx) *idx = at<int32_t>(workspace, L.idx);
    if (logw) *logw = at<float>(workspace, L.logw);
    return ABATT_OK;
}

abatt_status abatt_test_set(int hook, uint64_t value) {
    switch (hook) {
        case ABATT_TEST_WAIT_NS: g_wait_ns.store(value ? value : kWaitNs); return ABATT_OK;
        case ABATT_TEST_STALL: g_stall.store((uint32_t)value); return ABATT_OK;
    }
    return ABATT_ERR_INVALID_ARG;
}

abatt_status abatt_test_exp2_poly(const float *x, float *y, int64_t n, int degree, void *stream) {
    if (!x || !y || n < 0 || (degree != 3 && degree != 4)) return ABATT_ERR_INVALID_ARG;
    if (n == 0) return ABATT_OK;
    int sms = 0;
    abatt_status s = device_sms(&sms);
    if (s != ABATT_OK) return s;
    int64_t grid = (n + 511) / 512;
    if (grid > (int64_t)sms * 8) grid = (int64_t)sms * 8;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (degree == 3) exp2_poly_kernel<3><<<(unsigned)grid, 256, 0, st>>>(x, y, n);
    else exp2_poly_kernel<4><<<(unsigned)grid, 256, 0, st>>>(x, y, n);
    return cuda_status(cudaGetLastError());
}

abatt_status abatt_read_status(const void *workspace, uint32_t *flags, void *stream) {
    if (!workspace || !flags) return ABATT_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return ABATT_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, workspace, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess)
        return ABATT_ERR_CUDA;
    *flags = v;
    return v ? ABATT_ERR_DEVICE : ABATT_OK;
}

abatt_status abatt_clear_status(void *workspace, void *stream) {
    if (!workspace) return ABATT_ERR_INVALID_ARG;
    return cuda_status(
        cudaMemsetAsync(workspace, 0, sizeof(WsHeader), static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
