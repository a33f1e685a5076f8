// C ABI of libfavor.so (declared in include/favor.h). Single translation unit: the kernel files
// are included here so the device status word has one definition without relocatable code.
//
// Host responsibilities: argument validation before any launch, workspace carving, TMA tensor
// maps, and the launch sequence per call. Every step of the computation runs in the kernels.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "common.cuh"

#include "k_fp32.cu"
#include "k_keys_bidir.cu"
#include "k_query.cu"
#include "k_keys_wide.cu"
#include "k_causal.cu"
#include "k_gemm.cu"
#include "k_selftest.cu"
#include "k_decode.cu"

namespace favor {
namespace {

// ------------------------------------------------------------------------------- validation

bool shape_ok(const favor_shape *s) {
    if (s == nullptr) return false;
    if (s->B <= 0 || s->H <= 0 || s->L <= 0 || s->d <= 0 || s->m <= 0) return false;
    if (s->dtype != FAVOR_F32 && s->dtype != FAVOR_BF16) return false;
    if ((long long)s->B * s->H * s->L > (1ll << 31)) return false;
    return true;
}

// What the kernels implement for this shape (FAVOR_OK or FAVOR_ERR_UNSUPPORTED).
favor_status shape_supported(const favor_shape *s, int causal, int backward) {
    if (s->d != 64 && s->d != 128) return FAVOR_ERR_UNSUPPORTED;
    if ((long long)s->B * s->H > 65535) return FAVOR_ERR_UNSUPPORTED;
    if (s->dtype == FAVOR_F32) {
        if (s->m % 16 != 0 || s->m > 512) return FAVOR_ERR_UNSUPPORTED;
        return FAVOR_OK;
    }
    if (s->m != 128 && s->m != 256) return FAVOR_ERR_UNSUPPORTED;
    // the causal path (forward, and the backward that reads its context) is built for d = 64
    if (causal && s->d != 64) return FAVOR_ERR_UNSUPPORTED;
    return FAVOR_OK;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Share of feature exponentials on the FMA-pipe polynomial (percent) for a kernel whose default is
// dflt: 0 (or no opts) takes that default, 1..100 is used as given, a negative value puts every
// exponential on MUFU. Defaults measured on B200 (bidirectional d = 64, L = 4096): the query output
// kernel runs 1 us faster (of 40) with a quarter on the polynomial, the key kernel is best with none
// (and both lose from 37 % on); the other kernels keep everything on MUFU.
int opt_poly_pct(const favor_opts *o, int dflt) {
    const int v = o ? o->exp_poly_pct : 0;
    if (v == 0) return dflt;
    return v > 0 ? std::min(v, 100) : 0;
}
constexpr int kQueryPolyPct = 25;  // k_query_out, d = 64

int opt_feature_map(const favor_opts *o) { return o ? o->feature_map : FAVOR_MAP_POSITIVE; }

int opt_split_tiles(const favor_opts *o) {
    const int v = o ? o->split_tiles : 0;
    return v > 0 ? std::min(v, 64) : 8;
}

// -------------------------------------------------------------------------------- workspace

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Tokens per head whose causal outputs are recomputed at split precision (bf16 hi + lo operands,
// fp32 accumulation): the first outputs of a head average few values and are far larger than the
// head's RMS output, beyond what the fp16 chunk kernel resolves.
constexpr int kCausalExactPrefix = 512;
// Key columns of the prefix's masked score matrix: P rounded up to the 128-wide GEMM tile.
int prefix_cols(int P) { return (P + 127) & ~127; }

// Causal bf16 forward: per-key -|k|^2/2, the per-segment partial states of k_key_partials_wide
// ([S' | z'] columns feature-minor, per-feature stabilisers, per-warp maxima), the exclusive
// segment prefixes at the head reference, and the exact prefix's features and scores.
struct Bf16Layout {
    int BH, n_tiles, tiles_per_split, n_split, n_seg, P_exact, Ppad;
    size_t off_bias, off_head_max, off_part, off_part_D, off_part_amax, off_part_umax, off_seg_vmax, off_seg_S,
        off_seg_z, off_kref, off_pq[2], off_pk[2], off_pa[2], total;
};

Bf16Layout bf16_layout(const favor_shape *s, const favor_opts *o) {
    Bf16Layout l{};
    l.BH = s->B * s->H;
    l.n_tiles = (s->L + kTile - 1) / kTile;
    l.tiles_per_split = opt_split_tiles(o);
    l.n_split = (l.n_tiles + l.tiles_per_split - 1) / l.tiles_per_split;
    l.n_seg = l.BH * l.n_split;
    size_t off = 0;
    l.off_bias = off;
    off += align256((size_t)l.BH * s->L * 4);
    l.off_head_max = off;
    off += align256((size_t)l.BH * 4);
    l.off_part = off;
    off += align256((size_t)l.n_seg * (s->d + 1) * s->m * 4);
    l.off_part_D = off;
    off += align256((size_t)l.n_seg * s->m * 4);
    l.off_part_amax = off;
    off += align256((size_t)l.n_seg * 8 * 4);
    l.off_part_umax = off;
    off += align256((size_t)l.n_seg * 8 * 4);
    l.off_seg_vmax = off;
    off += align256((size_t)l.n_seg * 4);
    l.P_exact = std::min(s->L, kCausalExactPrefix);
    l.off_seg_S = off;
    off += align256((size_t)l.n_seg * s->m * s->d * 4);
    l.off_seg_z = off;
    off += align256((size_t)l.n_seg * s->m * 4);
    l.Ppad = prefix_cols(l.P_exact);
    l.off_kref = off;
    off += align256((size_t)l.BH * 4);
    for (int i = 0; i < 2; ++i) {
        l.off_pq[i] = off;
        off += align256((size_t)l.BH * l.P_exact * s->m * 2);
        l.off_pk[i] = off;
        off += align256((size_t)l.BH * l.P_exact * s->m * 2);
        l.off_pa[i] = off;
        off += align256((size_t)l.BH * l.P_exact * l.Ppad * 2);
    }
    l.total = off;
    return l;
}

// Bidirectional bf16 forward: per-run key maxima, per-run partial states [S | z] (feature-major
// columns), their largest magnitudes, and the per-head fp16 state images (unless a ctx holds them).
struct BidirLayout {
    Flat f;  // key tiles of the key-state kernel (128 tokens for d = 64, else 64)
    int BH;
    size_t off_part, off_D, off_amax, off_Dmax, off_state, total;
};

// Tokens per key tile: k_key_partials_wide (d = 64) takes 128, k_key_partials (d = 128) 64.
int bidir_key_tile(int d) { return d == 64 ? kWideTile : kKeyTile; }

BidirLayout bidir_layout(const favor_shape *s, bool state_in_ws) {
    BidirLayout l{};
    l.BH = s->B * s->H;
    l.f = make_flat(l.BH, s->L, num_sms(), bidir_key_tile(s->d));
    const size_t slots = (size_t)flat_slots(l.f, l.BH);
    size_t off = 0;
    l.off_part = off;
    off += align256(slots * (s->d + 1) * s->m * 4);
    l.off_D = off;
    off += align256(slots * s->m * 4);
    l.off_amax = off;
    off += align256(slots * 8 * 4);
    l.off_Dmax = off;
    off += align256(slots * 8 * 4);
    l.off_state = off;
    if (state_in_ws) off += align256((size_t)l.BH * state_floats(s->m, s->d) * 4);
    l.total = off;
    return l;
}


// Forward-to-backward context: per-head state blocks (the bidirectional fp16 state image, or the
// causal path's state), the causal per-key -|k|^2/2, and the per-head key reference C (log2
// units) the bidirectional backward's key features are taken against.
struct CtxLayout {
    size_t off_state, off_bias, off_kref, total;
};

CtxLayout ctx_layout(const favor_shape *s) {
    CtxLayout c{};
    const size_t BH = (size_t)s->B * s->H;
    c.off_state = 0;
    c.off_bias = align256(BH * state_floats(s->m, s->d) * 4);
    c.off_kref = c.off_bias + align256(BH * s->L * 4);
    c.total = c.off_kref + align256(BH * 4);
    return c;
}

size_t ctx_bytes(const favor_shape *s) { return ctx_layout(s).total; }

// bf16 bidirectional forward with a feature map other than the positive one (generalised
// attention, trigonometric features): phi(K), phi(Q) as hi/lo bf16 rows of mf features (m, or 2m
// for sin and cos), the state's token-split partial sums, and its hi/lo image [d+64][mf].
struct MapLayout {
    int BH, Np, mf, n_split, kt_split;
    size_t off_phk[2], off_phq[2], off_part, off_img[2], total;
};

MapLayout map_layout(const favor_shape *s, int map) {
    MapLayout l{};
    l.BH = s->B * s->H;
    l.Np = s->d + 64;
    l.mf = map == FAVOR_MAP_TRIG ? 2 * s->m : s->m;
    const int kt_total = (s->L + kGemmBK - 1) / kGemmBK;
    const int tiles = l.BH * (l.mf / 128);
    const int ns = std::max(1, std::min(kt_total, (2 * num_sms() + tiles - 1) / tiles));
    l.kt_split = (kt_total + ns - 1) / ns;
    l.n_split = (kt_total + l.kt_split - 1) / l.kt_split;
    const size_t tok = (size_t)l.BH * s->L;
    const size_t feat = align256(tok * l.mf * 2), img = align256((size_t)l.BH * l.Np * l.mf * 2);
    size_t off = 0;
    for (int i = 0; i < 2; ++i) { l.off_phk[i] = off; off += feat; }
    for (int i = 0; i < 2; ++i) { l.off_phq[i] = off; off += feat; }
    l.off_part = off; off += align256((size_t)l.BH * l.n_split * l.mf * l.Np * 4);
    for (int i = 0; i < 2; ++i) { l.off_img[i] = off; off += img; }
    l.total = off;
    return l;
}

// Sequence-parallel forward (bf16, bidirectional): per-feature offsets, phi(K) or phi(Q) hi/lo,
// the token-split partial state, its hi/lo image.
struct SpLayout {
    int BH, Np, n_split, kt_split;
    size_t off_c, off_phi[2], off_part, off_img[2], total;
};

SpLayout sp_layout(const favor_shape *s) {
    SpLayout l{};
    l.BH = s->B * s->H;
    l.Np = s->d + 64;
    const int kt_total = (s->L + kGemmBK - 1) / kGemmBK;
    const int tiles = l.BH * (s->m / 128);
    const int ns = std::max(1, std::min(kt_total, (2 * num_sms() + tiles - 1) / tiles));
    l.kt_split = (kt_total + ns - 1) / ns;
    l.n_split = (kt_total + l.kt_split - 1) / l.kt_split;
    const size_t tok = (size_t)l.BH * s->L;
    size_t off = 0;
    l.off_c = off; off += align256((size_t)s->m * 4);
    for (int i = 0; i < 2; ++i) { l.off_phi[i] = off; off += align256(tok * s->m * 2); }
    l.off_part = off; off += align256((size_t)l.BH * l.n_split * s->m * l.Np * 4);
    for (int i = 0; i < 2; ++i) { l.off_img[i] = off; off += align256((size_t)l.BH * l.Np * s->m * 2); }
    l.total = off;
    return l;
}

// bf16 causal backward: the same intermediates per token, the masked 128 x 128 diagonal tiles of
// every chunk, an fp32 scratch for the between-chunk terms, and per-chunk state images.
struct CausalBwdLayout {
    int BH, Np, nc;
    size_t off_phk[2], off_phq[2], off_gs[2], off_t[2], off_am[2], off_bm[2], off_x, off_rowsum, off_part, off_pimg[2],
        off_rimg[2], total;
};

CausalBwdLayout causal_bwd_layout(const favor_shape *s) {
    CausalBwdLayout l{};
    l.BH = s->B * s->H;
    l.Np = s->d + 64;
    l.nc = (s->L + kTile - 1) / kTile;
    const size_t tok = (size_t)l.BH * s->L;
    const size_t feat = align256(tok * s->m * 2), gsz = align256(tok * l.Np * 2), msk = align256(tok * kTile * 2);
    const size_t img = align256((size_t)l.BH * l.nc * l.Np * s->m * 2);
    size_t off = 0;
    for (int i = 0; i < 2; ++i) { l.off_phk[i] = off; off += feat; }
    for (int i = 0; i < 2; ++i) { l.off_phq[i] = off; off += feat; }
    for (int i = 0; i < 2; ++i) { l.off_gs[i] = off; off += gsz; }
    for (int i = 0; i < 2; ++i) { l.off_t[i] = off; off += feat; }
    for (int i = 0; i < 2; ++i) { l.off_am[i] = off; off += msk; }
    for (int i = 0; i < 2; ++i) { l.off_bm[i] = off; off += msk; }
    l.off_x = off; off += align256(tok * std::max(s->m, l.Np) * 4);
    l.off_rowsum = off; off += align256(tok * 8);  // two partial row sums per token
    l.off_part = off; off += align256((size_t)l.BH * l.nc * s->m * l.Np * 4);
    for (int i = 0; i < 2; ++i) { l.off_pimg[i] = off; off += img; }
    for (int i = 0; i < 2; ++i) { l.off_rimg[i] = off; off += img; }
    l.total = off;
    return l;
}

// bf16 bidirectional backward: hi/lo bf16 intermediates of the split-precision GEMM passes.
struct BwdLayout {
    int BH, Np, n_split, kt_split;
    size_t off_phk_hi, off_phk_lo, off_phq_hi, off_phq_lo, off_gs_hi, off_gs_lo, off_t_hi, off_t_lo, off_rowsum,
        off_part, off_sz_hi, off_sz_lo, off_g_hi, off_g_lo, total;
};

BwdLayout bwd_layout(const favor_shape *s) {
    BwdLayout l{};
    l.BH = s->B * s->H;
    l.Np = s->d + 64;
    // split the token reduction of the state sums over enough CTAs to fill the GPU about twice
    const int kt_total = (s->L + kGemmBK - 1) / kGemmBK;
    const int tiles = l.BH * (s->m / 128);
    int ns = std::max(1, std::min(kt_total, (2 * num_sms() + tiles - 1) / tiles));
    l.kt_split = (kt_total + ns - 1) / ns;
    l.n_split = (kt_total + l.kt_split - 1) / l.kt_split;
    const size_t tok = (size_t)l.BH * s->L;
    const size_t feat = align256(tok * s->m * 2), gsz = align256(tok * l.Np * 2), img = align256((size_t)l.BH * l.Np * s->m * 2);
    size_t off = 0;
    l.off_phk_hi = off; off += feat;
    l.off_phk_lo = off; off += feat;
    l.off_phq_hi = off; off += feat;
    l.off_phq_lo = off; off += feat;
    l.off_gs_hi = off; off += gsz;
    l.off_gs_lo = off; off += gsz;
    l.off_t_hi = off; off += feat;
    l.off_t_lo = off; off += feat;
    l.off_rowsum = off; off += align256(tok * 8);  // two partial row sums per token
    l.off_part = off; off += align256((size_t)l.BH * l.n_split * s->m * l.Np * 4);
    l.off_sz_hi = off; off += img;
    l.off_sz_lo = off; off += img;
    l.off_g_hi = off; off += img;
    l.off_g_lo = off; off += img;
    l.total = off;
    return l;
}

// ------------------------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

// [BH, L, d] bf16 tensor as a 3-D map (d, L, BH) with 64 x rows x 1 boxes, 128-byte swizzle;
// rows past L read as zeros.
bool make_token_map(CUtensorMap *map, const void *base, int BH, int L, int d, int rows = kTile) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)L * d * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [m, d] bf16 W as a 2-D map (d, m) with 64 x rows boxes (rows = m by default), 128-byte swizzle.
bool make_w_map(CUtensorMap *map, const void *base, int m, int d, int rows = 0) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)m};
    const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)(rows > 0 ? rows : m)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 [BH, L, d] output as a 3-D map (d, L, BH) with 32 x 32 x 1 boxes, 128-byte swizzle (the
// staging layout of the output epilogue); rows past L are not written.
bool make_out_map(CUtensorMap *map, void *base, int BH, int L, int d) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)L * d * 4};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// bf16 [batch][outer][inner] tensor as a 3-D map (inner, outer, batch) with 64 x box_outer x 1
// boxes, 128-byte swizzle; coordinates past the tensor read as zeros.
bool make_map3(CUtensorMap *map, const void *base, int inner, int outer, int batch, int box_outer) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)outer, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)inner * outer * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_outer, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

favor_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FAVOR_OK : FAVOR_ERR_CUDA; }

// Records the caller's timing event (2k before / 2k+1 after launch k), if one was supplied.
void record_stage(const favor_opts *o, int slot, cudaStream_t st) {
    if (o != nullptr && o->stage_events != nullptr && slot < 2 * FAVOR_MAX_STAGES && o->stage_events[slot] != nullptr)
        cudaEventRecord((cudaEvent_t)o->stage_events[slot], st);
}

// ---------------------------------------------------------------------------- bf16 forward

// Outputs of the first P = min(L, 512) tokens of every head at split precision, overwriting what the
// chunk kernel left there: phi(K) = 2^(u(k) log2e - C), phi(Q) = exp(Wq - rowmax) as hi/lo bf16,
// A = mask(phi(Q) phi(K)^T) (key j kept for j <= query i) as hi/lo, then out = num / den with
// [num | den] = A [V | 1]: four launches of the split-precision GEMM (k_gemm.cu).
favor_status causal_prefix(const favor_shape *s, const Bf16Layout &l, const void *Q, const void *K, const void *V,
                           const void *W, const float *kref, float *out, uint8_t *ws, const favor_opts *o,
                           cudaStream_t st) {
    const int BH = l.BH, L = s->L, d = s->d, m = s->m, P = l.P_exact, Pp = l.Ppad, Np = d + 64;
    uint16_t *pq[2], *pk[2], *pa[2];
    for (int i = 0; i < 2; ++i) {
        pq[i] = (uint16_t *)(ws + l.off_pq[i]);
        pk[i] = (uint16_t *)(ws + l.off_pk[i]);
        pa[i] = (uint16_t *)(ws + l.off_pa[i]);
    }
    CUtensorMap mK, mQ, mVn, mW, mPq[2], mPk[2], mPa[2];
    bool ok = make_map3(&mK, K, d, L, BH, 128) && make_map3(&mQ, Q, d, L, BH, 128) && make_map3(&mVn, V, d, L, BH, 64) &&
              make_map3(&mW, W, d, m, 1, m);
    for (int i = 0; ok && i < 2; ++i)
        ok = make_map3(&mPq[i], pq[i], m, P, BH, 128) && make_map3(&mPk[i], pk[i], m, P, BH, 128) &&
             make_map3(&mPa[i], pa[i], Pp, P, BH, 128);
    if (!ok) return FAVOR_ERR_CUDA;
    auto args = [&](int M, int N, int Kd) {
        GemmArgs a{};
        a.M = M;
        a.N = N;
        a.K = Kd;
        a.n_split = 1;
        a.kt_split = (Kd + kGemmBK - 1) / kGemmBK;
        a.a_batched = a.b_batched = 1;
        return a;
    };
    GemmArgs ak = args(P, m, d);
    ak.b_batched = 0;
    ak.ld_out = m;
    ak.out_hi = pk[0];
    ak.out_lo = pk[1];
    ak.kc = kref;
    record_stage(o, 6, st);
    cudaError_t e = launch_gemm_t<false, false, false, false, kEpiPhiKey>(mK, mK, mW, mW, ak, m, BH, st);
    if (e != cudaSuccess) return FAVOR_ERR_CUDA;
    GemmArgs aq = args(P, m, d);
    aq.b_batched = 0;
    aq.ld_out = m;
    aq.out_hi = pq[0];
    aq.out_lo = pq[1];
    e = launch_gemm_t<false, false, false, false, kEpiPhiQuery>(mQ, mQ, mW, mW, aq, m, BH, st);
    if (e != cudaSuccess) return FAVOR_ERR_CUDA;
    GemmArgs aa = args(P, Pp, m);
    aa.ld_out = Pp;
    aa.out_hi = pa[0];
    aa.out_lo = pa[1];
    e = launch_gemm_t<false, false, true, true, kEpiMask>(mPq[0], mPq[1], mPk[0], mPk[1], aa, 128, BH, st);
    if (e != cudaSuccess) return FAVOR_ERR_CUDA;
    GemmArgs ao = args(P, Np, Pp);
    ao.b_ones = 1;
    ao.ld_out = d;
    ao.out_f32 = out;
    ao.out_rows = L;
    ao.d = d;
    e = launch_gemm_t<false, true, true, false, kEpiOut>(mPa[0], mPa[1], mVn, mVn, ao, Np, BH, st);
    record_stage(o, 7, st);
    return e == cudaSuccess ? FAVOR_OK : FAVOR_ERR_CUDA;
}

favor_status fwd_bf16_bidir(const favor_shape *s, const void *Q, const void *K, const void *V, const void *W,
                            float *out, void *ctx, uint8_t *ws, size_t ws_bytes, const favor_opts *o, cudaStream_t st) {
    const BidirLayout l = bidir_layout(s, ctx == nullptr);
    if (ws_bytes < l.total) return FAVOR_ERR_WORKSPACE;
    CUtensorMap mQ, mK64, mV64, mW, mO;
    if (!make_token_map(&mQ, Q, l.BH, s->L, s->d) || !make_token_map(&mK64, K, l.BH, s->L, s->d, bidir_key_tile(s->d)) ||
        !make_token_map(&mV64, V, l.BH, s->L, s->d, bidir_key_tile(s->d)) || !make_w_map(&mW, W, s->m, s->d) ||
        !make_out_map(&mO, out, l.BH, s->L, s->d))
        return FAVOR_ERR_CUDA;
    float *part = (float *)(ws + l.off_part);
    float *partD = (float *)(ws + l.off_D);
    float *amax = (float *)(ws + l.off_amax);
    float *Dmax = (float *)(ws + l.off_Dmax);
    uint8_t *state = ctx ? (uint8_t *)ctx : ws + l.off_state;
    float *kref = ctx ? (float *)((uint8_t *)ctx + ctx_layout(s).off_kref) : nullptr;
    const size_t stride = state_floats(s->m, s->d) * 4;

    KeyStateParams2 ks{s->L, s->m, l.f, part, partD, amax, Dmax};
    record_stage(o, 0, st);
    cudaError_t e = s->d == 64 ? launch_key_partials_wide(mK64, mV64, mW, ks, opt_poly_pct(o, 0), st)
                               : launch_key_partials(mK64, mV64, mW, ks, s->d, opt_poly_pct(o, 0), st);
    record_stage(o, 1, st);
    if (e != cudaSuccess) return FAVOR_ERR_CUDA;
    ImageParams ip{s->m, s->d, l.f, part, partD, amax, Dmax, state, stride, kref};
    record_stage(o, 2, st);
    e = launch_state_image(ip, l.BH, st);
    record_stage(o, 3, st);
    if (e != cudaSuccess) return FAVOR_ERR_CUDA;
    QueryParams qp{s->L, s->d, s->m, l.BH, 0, state, stride};
    record_stage(o, 4, st);
    e = launch_query_out(mQ, mW, mO, qp, opt_poly_pct(o, s->d == 64 ? kQueryPolyPct : 0), st);
    record_stage(o, 5, st);
    return e == cudaSuccess ? FAVOR_OK : FAVOR_ERR_CUDA;
}

// Bidirectional forward with the ReLU or trigonometric feature map, as split-precision GEMM passes:
// phi(K) (hi/lo), [S | z] = phi(K)^T [V | 1] over token splits and reduced to a hi/lo image,
// phi(Q), then out = num / den from [num | den] = phi(Q) [S | z]. The 1/sqrt(m) of phi and, for the
// trigonometric queries, exp(|q|^2/2) are per-row constants that cancel in D^-1.
favor_status fwd_bf16_map(const favor_shape *s, int map, const void *Q, const void *K, const void *V, const void *W,
                          float *out, uint8_t *ws, size_t ws_bytes, const favor_opts *o, cudaStream_t st) {
    const MapLayout l = map_layout(s, map);
    if (ws_bytes < l.total) return FAVOR_ERR_WORKSPACE;
    const int BH = l.BH, L = s->L, d = s->d, m = s->m, mf = l.mf, Np = l.Np;
    uint16_t *phk[2], *phq[2], *img[2];
    for (int i = 0; i < 2; ++i) {
        phk[i] = (uint16_t *)(ws + l.off_phk[i]);
        phq[i] = (uint16_t *)(ws + l.off_phq[i]);
        img[i] = (uint16_t *)(ws + l.off_img[i]);
    }
    float *part = (float *)(ws + l.off_part);
    CUtensorMap mK, mQ, mVn, mW, mPhkT[2], mPhq[2], mImg[2];
    bool ok = make_map3(&mK, K, d, L, BH, 128) && make_map3(&mQ, Q, d, L, BH, 128) && make_map3(&mVn, V, d, L, BH, 64) &&
              make_map3(&mW, W, d, m, 1, m);
    for (int i = 0; ok && i < 2; ++i)
        ok = make_map3(&mPhkT[i], phk[i], mf, L, BH, 64) && make_map3(&mPhq[i], phq[i], mf, L, BH, 128) &&
             make_map3(&mImg[i], img[i], mf, Np, BH, Np);
    if (!ok) return FAVOR_ERR_CUDA;
    auto args = [&](int M, int N, int Kd) {
        GemmArgs a{};
        a.M = M;
        a.N = N;
        a.K = Kd;
        a.n_split = 1;
        a.kt_split = (Kd + kGemmBK - 1) / kGemmBK;
        a.a_batched = a.b_batched = 1;
        return a;
    };
    int stage = 0;
    cudaError_t e = cudaSuccess;
    auto run = [&](auto launch) {
        if (e != cudaSuccess) return;
        record_stage(o, 2 * stage, st);
        e = launch();
        record_stage(o, 2 * stage + 1, st);
        ++stage;
    };
    const bool trig = map == FAVOR_MAP_TRIG;
    GemmArgs ak = args(L, m, d);
    ak.b_batched = 0;
    ak.ld_out = mf;
    ak.out_hi = phk[0];
    ak.out_lo = phk[1];
    run([&] {
        return trig ? launch_gemm_t<false, false, false, false, kEpiTrigK>(mK, mK, mW, mW, ak, m, BH, st)
                    : launch_gemm_t<false, false, false, false, kEpiRelu>(mK, mK, mW, mW, ak, m, BH, st);
    });
    GemmArgs as = args(mf, Np, L);
    as.n_split = l.n_split;
    as.kt_split = l.kt_split;
    as.b_ones = 1;
    as.ld_out = Np;
    as.out_f32 = part;
    run([&] { return launch_gemm_t<true, true, true, false, kEpiPartial>(mPhkT[0], mPhkT[1], mVn, mVn, as, Np, BH, st); });
    run([&] { return launch_reduce_image(part, l.n_split, mf, Np, img[0], img[1], BH, st); });
    GemmArgs aq = args(L, m, d);
    aq.b_batched = 0;
    aq.ld_out = mf;
    aq.out_hi = phq[0];
    aq.out_lo = phq[1];
    run([&] {
        return trig ? launch_gemm_t<false, false, false, false, kEpiTrigQ>(mQ, mQ, mW, mW, aq, m, BH, st)
                    : launch_gemm_t<false, false, false, false, kEpiRelu>(mQ, mQ, mW, mW, aq, m, BH, st);
    });
    GemmArgs ao = args(L, Np, mf);
    ao.ld_out = d;
    ao.out_f32 = out;
    ao.d = d;
    run([&] { return launch_gemm_t<false, false, true, true, kEpiOut>(mPhq[0], mPhq[1], mImg[0], mImg[1], ao, Np, BH, st); });
    return cuda_status(e);
}

favor_status fwd_bf16(const favor_shape *s, const void *Q, const void *K, const void *V, const void *W, float *out,
                      void *ctx, uint8_t *ws, size_t ws_bytes, const favor_opts *o, cudaStream_t st, int causal) {
    const int map = opt_feature_map(o);
    if (map != FAVOR_MAP_POSITIVE) return fwd_bf16_map(s, map, Q, K, V, W, out, ws, ws_bytes, o, st);
    if (!causal) return fwd_bf16_bidir(s, Q, K, V, W, out, ctx, ws, ws_bytes, o, st);
    const Bf16Layout l = bf16_layout(s, o);
    if (ws_bytes < l.total) return FAVOR_ERR_WORKSPACE;
    CUtensorMap mQ, mK, mV, mW, mW128;
    if (!make_token_map(&mQ, Q, l.BH, s->L, s->d) || !make_token_map(&mK, K, l.BH, s->L, s->d) ||
        !make_token_map(&mV, V, l.BH, s->L, s->d) || !make_w_map(&mW, W, s->m, s->d) ||
        !make_w_map(&mW128, W, s->m, s->d, 128))
        return FAVOR_ERR_CUDA;
    // Per-key -|k|^2/2 goes straight into the context (after the state blocks) when one is kept.
    float *bias = ctx ? (float *)((uint8_t *)ctx + ctx_layout(s).off_bias) : (float *)(ws + l.off_bias);
    float *head_max = (float *)(ws + l.off_head_max);
    float *seg_S = (float *)(ws + l.off_seg_S);
    float *seg_z = (float *)(ws + l.off_seg_z);
    // the head's key reference in log2 units, for the exact prefix and (in the context) the backward
    float *kref = ctx ? (float *)((uint8_t *)ctx + ctx_layout(s).off_kref) : (float *)(ws + l.off_kref);

    // per-segment states (one pass over K and V; 128-token tiles, per-feature stabilisers)
    CUtensorMap mK128, mV128;
    if (!make_token_map(&mK128, K, l.BH, s->L, s->d, kWideTile) || !make_token_map(&mV128, V, l.BH, s->L, s->d, kWideTile))
        return FAVOR_ERR_CUDA;
    const int segs_per_cta = (l.n_seg + num_sms() - 1) / num_sms();
    Flat f{};
    f.nt = l.n_tiles;
    f.total = l.BH * l.n_tiles;
    float *part = (float *)(ws + l.off_part);
    KeyStateParams2 ks{s->L, s->m, f, part, (float *)(ws + l.off_part_D), (float *)(ws + l.off_part_amax),
                       (float *)(ws + l.off_part_umax)};
    uint32_t *seg_vmax = (uint32_t *)(ws + l.off_seg_vmax);
    const WideSegParams sgp{l.n_split, l.tiles_per_split, l.n_seg, segs_per_cta, bias, seg_vmax};
    record_stage(o, 0, st);
    cudaError_t e = launch_key_segments(mK128, mV128, mW, ks, sgp, opt_poly_pct(o, 0), st);
    record_stage(o, 1, st);
    if (e != cudaSuccess) return FAVOR_ERR_CUDA;
    SegScanParams sp{s->m, l.n_split, s->m / 128, part, (float *)(ws + l.off_part_D), (float *)(ws + l.off_part_umax),
                     seg_S, seg_z, head_max, kref};
    record_stage(o, 2, st);
    e = launch_segment_scan(sp, l.BH, st);
    record_stage(o, 3, st);
    if (e != cudaSuccess) return FAVOR_ERR_CUDA;
    ChunkParams cp{s->L, s->m, l.n_split, l.tiles_per_split, l.P_exact, l.BH * l.n_split, bias, head_max,
                   seg_S, seg_z, seg_vmax, out};
    record_stage(o, 4, st);
    e = launch_causal_chunk(mQ, mK, mV, mW128, cp, opt_poly_pct(o, 0), st);
    record_stage(o, 5, st);
    if (e != cudaSuccess) return FAVOR_ERR_CUDA;
    return causal_prefix(s, l, Q, K, V, W, kref, out, ws, o, st);
}

// ---------------------------------------------------------------------------- bf16 backward

// Bidirectional bf16 backward (W fixed) as split-precision GEMM passes. With
// phi(k) = 2^(u(k) log2e - C) (C: the head's key reference from the forward's context) and
// phi(q) = exp(W q - rowmax) (a per-row constant that cancels):
//   [S | z] = phi(K)^T [V | 1]                      (state, reduced over tokens)
//   [num | den] = phi(Q) [S | z] -> g = dO/den, s = -(dO . num/den)/den
//   dphi(Q) = [g | s] [S | z]^T, t = phi(Q) * dphi(Q), dQ = t W - Q rowsum(t)
//   [G | h] = phi(Q)^T [g | s]                      (reduced over tokens)
//   dV = phi(K) G,  dphi(K) = [V | 1] [G | h]^T, t = phi(K) * dphi(K), dK = t W - K rowsum(t)
// Every constant factor cancels (C between [S | z] and [G | h], the row maxima between [num | den]
// and [g | s]), so no rescaling is needed.
favor_status bwd_bf16_bidir(const favor_shape *s, const void *Q, const void *K, const void *V, const void *W,
                            const void *dout, const void *ctx, float *dQ, float *dK, float *dV, uint8_t *ws,
                            size_t ws_bytes, const favor_opts *o, cudaStream_t st) {
    const BwdLayout l = bwd_layout(s);
    if (ws_bytes < l.total) return FAVOR_ERR_WORKSPACE;
    const int BH = l.BH, L = s->L, d = s->d, m = s->m, Np = l.Np;
    auto at = [&](size_t off) { return (uint16_t *)(ws + off); };
    uint16_t *phk_hi = at(l.off_phk_hi), *phk_lo = at(l.off_phk_lo), *phq_hi = at(l.off_phq_hi),
             *phq_lo = at(l.off_phq_lo), *gs_hi = at(l.off_gs_hi), *gs_lo = at(l.off_gs_lo), *t_hi = at(l.off_t_hi),
             *t_lo = at(l.off_t_lo), *sz_hi = at(l.off_sz_hi), *sz_lo = at(l.off_sz_lo), *g_hi = at(l.off_g_hi),
             *g_lo = at(l.off_g_lo);
    float *rowsum = (float *)(ws + l.off_rowsum), *part = (float *)(ws + l.off_part);
    const float *kref = (const float *)((const uint8_t *)ctx + ctx_layout(s).off_kref);

    // token-major operands (box rows 128 for K-major A, 64 for the other reads)
    CUtensorMap mK, mQ, mV, mW_k, mW_n, mPhk[2], mPhkT[2], mPhq[2], mPhqT[2], mGs[2], mGsT[2], mT[2], mSzK[2],
        mSzN[2], mGK[2], mGN[2];
    bool ok = make_map3(&mK, K, d, L, BH, 128) && make_map3(&mQ, Q, d, L, BH, 128) && make_map3(&mV, V, d, L, BH, 128) &&
              make_map3(&mW_k, W, d, m, 1, m) && make_map3(&mW_n, W, d, m, 1, 64);
    uint16_t *phk[2] = {phk_hi, phk_lo}, *phq[2] = {phq_hi, phq_lo}, *gs[2] = {gs_hi, gs_lo}, *tt[2] = {t_hi, t_lo},
             *sz[2] = {sz_hi, sz_lo}, *gi[2] = {g_hi, g_lo};
    CUtensorMap mVn;
    ok = ok && make_map3(&mVn, V, d, L, BH, 64);
    for (int i = 0; ok && i < 2; ++i)
        ok = make_map3(&mPhk[i], phk[i], m, L, BH, 128) && make_map3(&mPhkT[i], phk[i], m, L, BH, 64) &&
             make_map3(&mPhq[i], phq[i], m, L, BH, 128) && make_map3(&mPhqT[i], phq[i], m, L, BH, 64) &&
             make_map3(&mGs[i], gs[i], Np, L, BH, 128) && make_map3(&mGsT[i], gs[i], Np, L, BH, 64) &&
             make_map3(&mT[i], tt[i], m, L, BH, 128) && make_map3(&mSzK[i], sz[i], m, Np, BH, Np) &&
             make_map3(&mSzN[i], sz[i], m, Np, BH, 64) && make_map3(&mGK[i], gi[i], m, Np, BH, d) &&
             make_map3(&mGN[i], gi[i], m, Np, BH, 64);
    if (!ok) return FAVOR_ERR_CUDA;

    int stage = 0;
    cudaError_t e = cudaSuccess;
    auto run = [&](auto launch) {
        if (e != cudaSuccess) return;
        record_stage(o, 2 * stage, st);
        e = launch();
        record_stage(o, 2 * stage + 1, st);
        ++stage;
    };
    auto args = [&](int M, int N, int Kd) {
        GemmArgs a{};
        a.M = M;
        a.N = N;
        a.K = Kd;
        a.n_split = 1;
        a.kt_split = (Kd + kGemmBK - 1) / kGemmBK;
        a.a_batched = a.b_batched = 1;
        return a;
    };
    // 1. phi(K)
    GemmArgs a1 = args(L, m, d);
    a1.b_batched = 0;
    a1.ld_out = m;
    a1.out_hi = phk_hi;
    a1.out_lo = phk_lo;
    a1.kc = kref;
    run([&] { return launch_gemm_t<false, false, false, false, kEpiPhiKey>(mK, mK, mW_k, mW_k, a1, m, BH, st); });
    // 2. [S | z] partial sums over token splits, 3. reduced to the hi/lo image [Np][m]
    GemmArgs a2 = args(m, Np, L);
    a2.n_split = l.n_split;
    a2.kt_split = l.kt_split;
    a2.b_ones = 1;
    a2.ld_out = Np;
    a2.out_f32 = part;
    run([&] { return launch_gemm_t<true, true, true, false, kEpiPartial>(mPhkT[0], mPhkT[1], mVn, mVn, a2, Np, BH, st); });
    run([&] { return launch_reduce_image(part, l.n_split, m, Np, sz_hi, sz_lo, BH, st); });
    // 4. phi(Q)
    GemmArgs a4 = args(L, m, d);
    a4.b_batched = 0;
    a4.ld_out = m;
    a4.out_hi = phq_hi;
    a4.out_lo = phq_lo;
    run([&] { return launch_gemm_t<false, false, false, false, kEpiPhiQuery>(mQ, mQ, mW_k, mW_k, a4, m, BH, st); });
    // 5. [num | den] -> [g | s]
    GemmArgs a5 = args(L, Np, m);
    a5.ld_out = Np;
    a5.out_hi = gs_hi;
    a5.out_lo = gs_lo;
    a5.side_hi = (const uint16_t *)dout;
    a5.ld_side = d;
    a5.d = d;
    run([&] { return launch_gemm_t<false, false, true, true, kEpiGS>(mPhq[0], mPhq[1], mSzK[0], mSzK[1], a5, Np, BH, st); });
    // 6. dphi(Q) -> t = phi(Q) * dphi(Q) and its row sums
    GemmArgs a6 = args(L, m, Np);
    a6.ld_out = m;
    a6.out_hi = t_hi;
    a6.out_lo = t_lo;
    a6.rowsum = rowsum;
    a6.side_hi = phq_hi;
    a6.side_lo = phq_lo;
    a6.ld_side = m;
    run([&] { return launch_gemm_t<false, true, true, true, kEpiT>(mGs[0], mGs[1], mSzN[0], mSzN[1], a6, m, BH, st); });
    // 7. dQ = t W - Q rowsum(t)
    GemmArgs a7 = args(L, d, m);
    a7.b_batched = 0;
    a7.ld_out = d;
    a7.out_f32 = dQ;
    a7.rowsum = rowsum;
    a7.side_hi = (const uint16_t *)Q;
    a7.ld_side = d;
    run([&] { return launch_gemm_t<false, true, true, false, kEpiDX>(mT[0], mT[1], mW_n, mW_n, a7, d, BH, st); });
    // 8. [G | h] partial sums over token splits, 9. reduced to the hi/lo image [Np][m]
    GemmArgs a8 = args(m, Np, L);
    a8.n_split = l.n_split;
    a8.kt_split = l.kt_split;
    a8.ld_out = Np;
    a8.out_f32 = part;
    run([&] { return launch_gemm_t<true, true, true, true, kEpiPartial>(mPhqT[0], mPhqT[1], mGsT[0], mGsT[1], a8, Np, BH, st); });
    run([&] { return launch_reduce_image(part, l.n_split, m, Np, g_hi, g_lo, BH, st); });
    // 10. dV = phi(K) G
    GemmArgs a10 = args(L, d, m);
    a10.ld_out = d;
    a10.out_f32 = dV;
    run([&] { return launch_gemm_t<false, false, true, true, kEpiF32>(mPhk[0], mPhk[1], mGK[0], mGK[1], a10, d, BH, st); });
    // 11. dphi(K) = [V | 1] [G | h]^T -> t = phi(K) * dphi(K) and its row sums
    GemmArgs a11 = args(L, m, Np);
    a11.a_ones = 1;
    a11.ld_out = m;
    a11.out_hi = t_hi;
    a11.out_lo = t_lo;
    a11.rowsum = rowsum;
    a11.side_hi = phk_hi;
    a11.side_lo = phk_lo;
    a11.ld_side = m;
    run([&] { return launch_gemm_t<false, true, false, true, kEpiT>(mV, mV, mGN[0], mGN[1], a11, m, BH, st); });
    // 12. dK = t W - K rowsum(t)
    GemmArgs a12 = args(L, d, m);
    a12.b_batched = 0;
    a12.ld_out = d;
    a12.out_f32 = dK;
    a12.rowsum = rowsum;
    a12.side_hi = (const uint16_t *)K;
    a12.ld_side = d;
    run([&] { return launch_gemm_t<false, true, true, false, kEpiDX>(mT[0], mT[1], mW_n, mW_n, a12, d, BH, st); });
    return cuda_status(e);
}

// Causal bf16 backward (W fixed) as split-precision GEMM passes over 128-token chunks c (one GEMM
// M tile each). With P_c = sum_{j < 128c} phi(k_j) [v_j | 1]^T (exclusive prefix over chunks) and
// R_c = sum_{i >= 128(c+1)} phi(q_i) [g_i | s_i]^T (exclusive suffix), and the chunk's masked tiles
// A = mask(phi(Q_c) phi(K_c)^T), B = mask([g | s]_c [V | 1]_c^T) (column j kept for j <= row i):
//   [num | den] = phi(Q_c) P_c + A [V | 1]_c             -> g, s
//   dphi(Q)     = [g | s]_c P_c^T + B phi(K_c)           -> t, dQ = t W - Q rowsum(t)
//   dV          = phi(K_c) R_c[:, :d] + A^T g_c
//   dphi(K)     = [V | 1]_c R_c^T + B^T phi(Q_c)         -> t, dK = t W - K rowsum(t)
// (the suffix sums G_j, h_j over i >= j of the masked recurrence, split at the chunk boundary).
favor_status bwd_bf16_causal(const favor_shape *s, const void *Q, const void *K, const void *V, const void *W,
                             const void *dout, const void *ctx, float *dQ, float *dK, float *dV, uint8_t *ws,
                             size_t ws_bytes, const favor_opts *o, cudaStream_t st) {
    const CausalBwdLayout l = causal_bwd_layout(s);
    if (ws_bytes < l.total) return FAVOR_ERR_WORKSPACE;
    const int BH = l.BH, L = s->L, d = s->d, m = s->m, Np = l.Np, nc = l.nc;
    auto at = [&](size_t off) { return (uint16_t *)(ws + off); };
    uint16_t *phk[2] = {at(l.off_phk[0]), at(l.off_phk[1])}, *phq[2] = {at(l.off_phq[0]), at(l.off_phq[1])},
             *gs[2] = {at(l.off_gs[0]), at(l.off_gs[1])}, *tt[2] = {at(l.off_t[0]), at(l.off_t[1])},
             *am[2] = {at(l.off_am[0]), at(l.off_am[1])}, *bm[2] = {at(l.off_bm[0]), at(l.off_bm[1])},
             *pimg[2] = {at(l.off_pimg[0]), at(l.off_pimg[1])}, *rimg[2] = {at(l.off_rimg[0]), at(l.off_rimg[1])};
    float *X = (float *)(ws + l.off_x), *rowsum = (float *)(ws + l.off_rowsum), *part = (float *)(ws + l.off_part);
    const float *kref = (const float *)((const uint8_t *)ctx + ctx_layout(s).off_kref);

    CUtensorMap mK, mQ, mV, mVn, mW_k, mW_n, mPhk[2], mPhkT[2], mPhq[2], mPhqT[2], mGs[2], mGsT[2], mT[2], mAm[2],
        mAmT[2], mBm[2], mBmT[2], mPK[2], mPN[2], mRK[2], mRN[2];
    bool ok = make_map3(&mK, K, d, L, BH, 128) && make_map3(&mQ, Q, d, L, BH, 128) && make_map3(&mV, V, d, L, BH, 128) &&
              make_map3(&mVn, V, d, L, BH, 64) && make_map3(&mW_k, W, d, m, 1, m) && make_map3(&mW_n, W, d, m, 1, 64);
    for (int i = 0; ok && i < 2; ++i)
        ok = make_map3(&mPhk[i], phk[i], m, L, BH, 128) && make_map3(&mPhkT[i], phk[i], m, L, BH, 64) &&
             make_map3(&mPhq[i], phq[i], m, L, BH, 128) && make_map3(&mPhqT[i], phq[i], m, L, BH, 64) &&
             make_map3(&mGs[i], gs[i], Np, L, BH, 128) && make_map3(&mGsT[i], gs[i], Np, L, BH, 64) &&
             make_map3(&mT[i], tt[i], m, L, BH, 128) && make_map3(&mAm[i], am[i], kTile, L, BH, 128) &&
             make_map3(&mAmT[i], am[i], kTile, L, BH, 64) && make_map3(&mBm[i], bm[i], kTile, L, BH, 128) &&
             make_map3(&mBmT[i], bm[i], kTile, L, BH, 64) && make_map3(&mPK[i], pimg[i], m, Np, BH * nc, Np) &&
             make_map3(&mPN[i], pimg[i], m, Np, BH * nc, 64) && make_map3(&mRK[i], rimg[i], m, Np, BH * nc, d) &&
             make_map3(&mRN[i], rimg[i], m, Np, BH * nc, 64);
    if (!ok) return FAVOR_ERR_CUDA;

    int stage = 0;
    cudaError_t e = cudaSuccess;
    auto run = [&](auto launch) {
        if (e != cudaSuccess) return;
        record_stage(o, 2 * stage, st);
        e = launch();
        record_stage(o, 2 * stage + 1, st);
        ++stage;
    };
    auto args = [&](int M, int N, int Kd) {
        GemmArgs a{};
        a.M = M;
        a.N = N;
        a.K = Kd;
        a.n_split = 1;
        a.kt_split = (Kd + kGemmBK - 1) / kGemmBK;
        a.a_batched = a.b_batched = 1;
        return a;
    };
    // phi(K), phi(Q)
    GemmArgs ak = args(L, m, d);
    ak.b_batched = 0;
    ak.ld_out = m;
    ak.out_hi = phk[0];
    ak.out_lo = phk[1];
    ak.kc = kref;
    run([&] { return launch_gemm_t<false, false, false, false, kEpiPhiKey>(mK, mK, mW_k, mW_k, ak, m, BH, st); });
    GemmArgs aq = args(L, m, d);
    aq.b_batched = 0;
    aq.ld_out = m;
    aq.out_hi = phq[0];
    aq.out_lo = phq[1];
    run([&] { return launch_gemm_t<false, false, false, false, kEpiPhiQuery>(mQ, mQ, mW_k, mW_k, aq, m, BH, st); });
    // per-chunk key states phi(K_c)^T [V | 1]_c, exclusive prefix images P_c
    GemmArgs as = args(m, Np, L);
    as.n_split = nc;
    as.kt_split = kTile / kGemmBK;
    as.b_ones = 1;
    as.ld_out = Np;
    as.out_f32 = part;
    run([&] { return launch_gemm_t<true, true, true, false, kEpiPartial>(mPhkT[0], mPhkT[1], mVn, mVn, as, Np, BH, st); });
    run([&] { return launch_scan_image(part, nc, m, Np, 0, pimg[0], pimg[1], BH, st); });
    // A = mask(phi(Q_c) phi(K_c)^T)
    GemmArgs aa = args(L, kTile, m);
    aa.b_nofs = 1;
    aa.ld_out = kTile;
    aa.out_hi = am[0];
    aa.out_lo = am[1];
    run([&] { return launch_gemm_t<false, false, true, true, kEpiMask>(mPhq[0], mPhq[1], mPhk[0], mPhk[1], aa, kTile, BH, st); });
    // [num | den]: phi(Q_c) P_c into X, then A [V | 1]_c + X -> [g | s]
    GemmArgs an = args(L, Np, m);
    an.b_chunk = 1;
    an.n_chunks = nc;
    an.ld_out = Np;
    an.out_f32 = X;
    run([&] { return launch_gemm_t<false, false, true, true, kEpiF32>(mPhq[0], mPhq[1], mPK[0], mPK[1], an, Np, BH, st); });
    GemmArgs ag = args(L, Np, kTile);
    ag.b_kofs = 1;
    ag.b_ones = 1;
    ag.addend = X;
    ag.ld_add = Np;
    ag.ld_out = Np;
    ag.out_hi = gs[0];
    ag.out_lo = gs[1];
    ag.side_hi = (const uint16_t *)dout;
    ag.ld_side = d;
    ag.d = d;
    run([&] { return launch_gemm_t<false, true, true, false, kEpiGS>(mAm[0], mAm[1], mVn, mVn, ag, Np, BH, st); });
    // B = mask([g | s]_c [V | 1]_c^T)
    GemmArgs ab = args(L, kTile, Np);
    ab.b_nofs = 1;
    ab.b_ones_k = 1;
    ab.ld_out = kTile;
    ab.out_hi = bm[0];
    ab.out_lo = bm[1];
    run([&] { return launch_gemm_t<false, false, true, false, kEpiMask>(mGs[0], mGs[1], mV, mV, ab, kTile, BH, st); });
    // dphi(Q): [g | s]_c P_c^T into X, then B phi(K_c) + X -> t, rowsum(t)
    GemmArgs ad = args(L, m, Np);
    ad.b_chunk = 1;
    ad.n_chunks = nc;
    ad.ld_out = m;
    ad.out_f32 = X;
    run([&] { return launch_gemm_t<false, true, true, true, kEpiF32>(mGs[0], mGs[1], mPN[0], mPN[1], ad, m, BH, st); });
    GemmArgs at2 = args(L, m, kTile);
    at2.b_kofs = 1;
    at2.addend = X;
    at2.ld_add = m;
    at2.ld_out = m;
    at2.out_hi = tt[0];
    at2.out_lo = tt[1];
    at2.rowsum = rowsum;
    at2.side_hi = phq[0];
    at2.side_lo = phq[1];
    at2.ld_side = m;
    run([&] { return launch_gemm_t<false, true, true, true, kEpiT>(mBm[0], mBm[1], mPhkT[0], mPhkT[1], at2, m, BH, st); });
    // dQ = t W - Q rowsum(t)
    GemmArgs aqq = args(L, d, m);
    aqq.b_batched = 0;
    aqq.ld_out = d;
    aqq.out_f32 = dQ;
    aqq.rowsum = rowsum;
    aqq.side_hi = (const uint16_t *)Q;
    aqq.ld_side = d;
    run([&] { return launch_gemm_t<false, true, true, false, kEpiDX>(mT[0], mT[1], mW_n, mW_n, aqq, d, BH, st); });
    // per-chunk query sums phi(Q_c)^T [g | s]_c, exclusive suffix images R_c
    GemmArgs ar = args(m, Np, L);
    ar.n_split = nc;
    ar.kt_split = kTile / kGemmBK;
    ar.ld_out = Np;
    ar.out_f32 = part;
    run([&] { return launch_gemm_t<true, true, true, true, kEpiPartial>(mPhqT[0], mPhqT[1], mGsT[0], mGsT[1], ar, Np, BH, st); });
    run([&] { return launch_scan_image(part, nc, m, Np, 1, rimg[0], rimg[1], BH, st); });
    // dV: phi(K_c) R_c[:, :d] into X, then A^T g_c + X
    GemmArgs av = args(L, d, m);
    av.b_chunk = 1;
    av.n_chunks = nc;
    av.ld_out = d;
    av.out_f32 = X;
    run([&] { return launch_gemm_t<false, false, true, true, kEpiF32>(mPhk[0], mPhk[1], mRK[0], mRK[1], av, d, BH, st); });
    GemmArgs av2 = args(L, d, kTile);
    av2.a_kofs = 1;
    av2.a_mlocal = 1;
    av2.b_kofs = 1;
    av2.addend = X;
    av2.ld_add = d;
    av2.ld_out = d;
    av2.out_f32 = dV;
    run([&] { return launch_gemm_t<true, true, true, true, kEpiF32>(mAmT[0], mAmT[1], mGsT[0], mGsT[1], av2, d, BH, st); });
    // dphi(K): [V | 1]_c R_c^T into X, then B^T phi(Q_c) + X -> t, rowsum(t)
    GemmArgs ae = args(L, m, Np);
    ae.a_ones = 1;
    ae.b_chunk = 1;
    ae.n_chunks = nc;
    ae.ld_out = m;
    ae.out_f32 = X;
    run([&] { return launch_gemm_t<false, true, false, true, kEpiF32>(mV, mV, mRN[0], mRN[1], ae, m, BH, st); });
    GemmArgs ak2 = args(L, m, kTile);
    ak2.a_kofs = 1;
    ak2.a_mlocal = 1;
    ak2.b_kofs = 1;
    ak2.addend = X;
    ak2.ld_add = m;
    ak2.ld_out = m;
    ak2.out_hi = tt[0];
    ak2.out_lo = tt[1];
    ak2.rowsum = rowsum;
    ak2.side_hi = phk[0];
    ak2.side_lo = phk[1];
    ak2.ld_side = m;
    run([&] { return launch_gemm_t<true, true, true, true, kEpiT>(mBmT[0], mBmT[1], mPhqT[0], mPhqT[1], ak2, m, BH, st); });
    // dK = t W - K rowsum(t)
    GemmArgs akk = args(L, d, m);
    akk.b_batched = 0;
    akk.ld_out = d;
    akk.out_f32 = dK;
    akk.rowsum = rowsum;
    akk.side_hi = (const uint16_t *)K;
    akk.ld_side = d;
    run([&] { return launch_gemm_t<false, true, true, false, kEpiDX>(mT[0], mT[1], mW_n, mW_n, akk, d, BH, st); });
    return cuda_status(e);
}

}  // namespace
}  // namespace favor

using namespace favor;

extern "C" const char *favor_status_string(favor_status st) {
    switch (st) {
        case FAVOR_OK: return "FAVOR_OK";
        case FAVOR_ERR_INVALID_ARG: return "FAVOR_ERR_INVALID_ARG: null pointer or invalid size";
        case FAVOR_ERR_UNSUPPORTED: return "FAVOR_ERR_UNSUPPORTED: valid arguments outside the implemented cases";
        case FAVOR_ERR_CUDA: return "FAVOR_ERR_CUDA: a CUDA runtime or driver call failed";
        case FAVOR_ERR_TIMEOUT: return "FAVOR_ERR_TIMEOUT: a bounded device-side wait gave up";
        case FAVOR_ERR_WORKSPACE: return "FAVOR_ERR_WORKSPACE: workspace or ctx missing or too small";
    }
    return "FAVOR: unknown status";
}

extern "C" size_t favor_workspace_size(const favor_shape *s, int causal, int backward, const favor_opts *o) {
    if (!shape_ok(s) || (causal != 0 && causal != 1)) return 0;
    if (shape_supported(s, causal, backward) != FAVOR_OK) return 0;
    const int map = opt_feature_map(o);
    if (map != FAVOR_MAP_POSITIVE) {
        if (map != FAVOR_MAP_RELU && map != FAVOR_MAP_TRIG) return 0;
        if (s->dtype != FAVOR_BF16 || causal || backward) return 0;
        return map_layout(s, map).total;
    }
    if (s->dtype == FAVOR_F32) return align256(f32_workspace_floats(s->B * s->H, s->L, s->d, s->m) * 4);
    if (backward) return causal ? causal_bwd_layout(s).total : bwd_layout(s).total;
    if (!causal) return bidir_layout(s, true).total;
    return bf16_layout(s, o).total;
}

extern "C" size_t favor_ctx_size(const favor_shape *s, int causal) {
    if (!shape_ok(s) || (causal != 0 && causal != 1)) return 0;
    return ctx_bytes(s);
}

extern "C" favor_status favor_fwd(const favor_shape *s, const void *Q, const void *K, const void *V, const void *W,
                                  int causal, float *out, void *ctx, void *workspace, size_t ws_bytes,
                                  const favor_opts *o, void *stream) {
    if (!shape_ok(s) || Q == nullptr || K == nullptr || V == nullptr || W == nullptr || out == nullptr ||
        (causal != 0 && causal != 1))
        return FAVOR_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(W) || !aligned16(out))
        return FAVOR_ERR_INVALID_ARG;
    const favor_status sup = shape_supported(s, causal, 0);
    if (sup != FAVOR_OK) return sup;
    const int map = opt_feature_map(o);
    if (map != FAVOR_MAP_POSITIVE &&
        ((map != FAVOR_MAP_RELU && map != FAVOR_MAP_TRIG) || s->dtype != FAVOR_BF16 || causal))
        return FAVOR_ERR_UNSUPPORTED;
    if (workspace == nullptr || ((uintptr_t)workspace & 255u) != 0) return FAVOR_ERR_WORKSPACE;
    if (ctx != nullptr && ((uintptr_t)ctx & 255u) != 0) return FAVOR_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    if (s->dtype == FAVOR_F32) {
        if (ws_bytes < favor_workspace_size(s, causal, 0, o)) return FAVOR_ERR_WORKSPACE;
        F32Params p{s->L, s->d, s->m, (const float *)Q, (const float *)K, (const float *)V, (const float *)W,
                    nullptr, nullptr, out, nullptr, nullptr, nullptr, (float *)workspace};
        return cuda_status(launch_f32(p, s->B * s->H, causal != 0, false, st));
    }
    return fwd_bf16(s, Q, K, V, W, out, ctx, (uint8_t *)workspace, ws_bytes, o, st, causal);
}

extern "C" favor_status favor_bwd(const favor_shape *s, const void *Q, const void *K, const void *V, const void *W,
                                  const float *out, const void *dout, const void *ctx, int causal, float *dQ,
                                  float *dK, float *dV, void *workspace, size_t ws_bytes, const favor_opts *o,
                                  void *stream) {
    if (!shape_ok(s) || Q == nullptr || K == nullptr || V == nullptr || W == nullptr || out == nullptr ||
        dout == nullptr || dQ == nullptr || dK == nullptr || dV == nullptr || (causal != 0 && causal != 1))
        return FAVOR_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(W) || !aligned16(out) || !aligned16(dout) ||
        !aligned16(dQ) || !aligned16(dK) || !aligned16(dV))
        return FAVOR_ERR_INVALID_ARG;
    const favor_status sup = shape_supported(s, causal, 1);
    if (sup != FAVOR_OK) return sup;
    if (opt_feature_map(o) != FAVOR_MAP_POSITIVE) return FAVOR_ERR_UNSUPPORTED;
    if (workspace == nullptr || ((uintptr_t)workspace & 255u) != 0) return FAVOR_ERR_WORKSPACE;
    if (ws_bytes < favor_workspace_size(s, causal, 1, o)) return FAVOR_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    if (s->dtype == FAVOR_BF16) {
        // the key reference of the forward's context keeps the backward's key features in range
        if (ctx == nullptr || ((uintptr_t)ctx & 255u) != 0) return FAVOR_ERR_WORKSPACE;
        uint8_t *ws = (uint8_t *)workspace;
        return causal ? bwd_bf16_causal(s, Q, K, V, W, dout, ctx, dQ, dK, dV, ws, ws_bytes, o, st)
                      : bwd_bf16_bidir(s, Q, K, V, W, dout, ctx, dQ, dK, dV, ws, ws_bytes, o, st);
    }
    F32Params p{s->L, s->d, s->m, (const float *)Q, (const float *)K, (const float *)V, (const float *)W,
                out, (const float *)dout, nullptr, dQ, dK, dV, (float *)workspace};
    return cuda_status(launch_f32(p, s->B * s->H, causal != 0, true, st));
}

extern "C" favor_status favor_sync_status(void *stream) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return FAVOR_ERR_CUDA;
    int v = FAVOR_OK;
    if (cudaMemcpyFromSymbol(&v, favor::g_status, sizeof(int)) != cudaSuccess) return FAVOR_ERR_CUDA;
    if (v != FAVOR_OK) {
        const int zero = FAVOR_OK;
        if (cudaMemcpyToSymbol(favor::g_status, &zero, sizeof(int)) != cudaSuccess) return FAVOR_ERR_CUDA;
    }
    return (favor_status)v;
}

extern "C" size_t favor_decode_state_size(const favor_shape *s) {
    if (!shape_ok(s) || (s->d != 64 && s->d != 128) || s->m % 32 != 0 || s->m > 256) return 0;
    return (size_t)s->B * s->H * ((size_t)s->d * s->m + 2 * (size_t)s->m) * 4;
}

extern "C" favor_status favor_decode_step(const favor_shape *s, const void *q, const void *k, const void *v,
                                          const void *W, float *state, float *out, void *stream) {
    if (!shape_ok(s) || s->L != 1 || q == nullptr || k == nullptr || v == nullptr || W == nullptr ||
        state == nullptr || out == nullptr)
        return FAVOR_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(W) || !aligned16(state) || !aligned16(out))
        return FAVOR_ERR_INVALID_ARG;
    if ((s->d != 64 && s->d != 128) || s->m % 32 != 0 || s->m > 256 || (long long)s->B * s->H > (1ll << 31) - 1)
        return FAVOR_ERR_UNSUPPORTED;
    DecodeParams p{s->B * s->H, s->m, s->dtype == FAVOR_BF16 ? 1 : 0, q, k, v, W, state, out};
    return cuda_status(launch_decode_step(p, s->d, (cudaStream_t)stream));
}

// ------------------------------------------------------------------ sequence-parallel forward

namespace favor {
namespace {

favor_status sp_check(const favor_shape *s, const void *a, const void *b, const void *c, const void *d, const void *e,
                      void *ws) {
    if (!shape_ok(s) || a == nullptr || b == nullptr || c == nullptr || d == nullptr || e == nullptr)
        return FAVOR_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(b) || !aligned16(c) || !aligned16(d) || !aligned16(e)) return FAVOR_ERR_INVALID_ARG;
    if (s->dtype != FAVOR_BF16 || (s->d != 64 && s->d != 128) || (s->m != 128 && s->m != 256) ||
        (long long)s->B * s->H > 65535)
        return FAVOR_ERR_UNSUPPORTED;
    if (ws == nullptr || ((uintptr_t)ws & 255u) != 0) return FAVOR_ERR_WORKSPACE;
    return FAVOR_OK;
}

GemmArgs sp_args(int M, int N, int Kd) {
    GemmArgs a{};
    a.M = M;
    a.N = N;
    a.K = Kd;
    a.n_split = 1;
    a.kt_split = (Kd + kGemmBK - 1) / kGemmBK;
    a.a_batched = a.b_batched = 1;
    return a;
}

}  // namespace
}  // namespace favor

extern "C" size_t favor_sp_state_size(const favor_shape *s) {
    if (!shape_ok(s)) return 0;
    return (size_t)s->B * s->H * s->m * (s->d + 64) * 4;
}

extern "C" size_t favor_sp_workspace_size(const favor_shape *s) {
    if (!shape_ok(s) || s->dtype != FAVOR_BF16 || (s->d != 64 && s->d != 128) || (s->m != 128 && s->m != 256))
        return 0;
    return sp_layout(s).total;
}

extern "C" favor_status favor_sp_state(const favor_shape *s, const void *K, const void *V, const void *W, float *state,
                                       void *workspace, size_t ws_bytes, void *stream) {
    const favor_status chk = sp_check(s, K, V, W, state, K, workspace);
    if (chk != FAVOR_OK) return chk;
    const SpLayout l = sp_layout(s);
    if (ws_bytes < l.total) return FAVOR_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t *ws = (uint8_t *)workspace;
    const int BH = l.BH, L = s->L, d = s->d, m = s->m, Np = l.Np;
    float *c = (float *)(ws + l.off_c), *part = (float *)(ws + l.off_part);
    uint16_t *phi[2] = {(uint16_t *)(ws + l.off_phi[0]), (uint16_t *)(ws + l.off_phi[1])};
    CUtensorMap mK, mVn, mW, mPhT[2];
    bool ok = make_map3(&mK, K, d, L, BH, 128) && make_map3(&mVn, V, d, L, BH, 64) && make_map3(&mW, W, d, m, 1, m);
    for (int i = 0; ok && i < 2; ++i) ok = make_map3(&mPhT[i], phi[i], m, L, BH, 64);
    if (!ok) return FAVOR_ERR_CUDA;
    if (launch_feature_offsets(W, m, d, c, st) != cudaSuccess) return FAVOR_ERR_CUDA;
    GemmArgs ak = sp_args(L, m, d);
    ak.b_batched = 0;
    ak.ld_out = m;
    ak.out_hi = phi[0];
    ak.out_lo = phi[1];
    ak.colbias = c;
    if (launch_gemm_t<false, false, false, false, kEpiPhiKey>(mK, mK, mW, mW, ak, m, BH, st) != cudaSuccess)
        return FAVOR_ERR_CUDA;
    GemmArgs as = sp_args(m, Np, L);
    as.n_split = l.n_split;
    as.kt_split = l.kt_split;
    as.b_ones = 1;
    as.ld_out = Np;
    as.out_f32 = part;
    if (launch_gemm_t<true, true, true, false, kEpiPartial>(mPhT[0], mPhT[1], mVn, mVn, as, Np, BH, st) != cudaSuccess)
        return FAVOR_ERR_CUDA;
    return cuda_status(launch_sum_partials(part, l.n_split, (size_t)m * Np, state, BH, st));
}

extern "C" favor_status favor_sp_output(const favor_shape *s, const void *Q, const void *W, const float *state,
                                        float *out, void *workspace, size_t ws_bytes, void *stream) {
    const favor_status chk = sp_check(s, Q, W, state, out, Q, workspace);
    if (chk != FAVOR_OK) return chk;
    const SpLayout l = sp_layout(s);
    if (ws_bytes < l.total) return FAVOR_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t *ws = (uint8_t *)workspace;
    const int BH = l.BH, L = s->L, d = s->d, m = s->m, Np = l.Np;
    float *c = (float *)(ws + l.off_c);
    uint16_t *phi[2] = {(uint16_t *)(ws + l.off_phi[0]), (uint16_t *)(ws + l.off_phi[1])};
    uint16_t *img[2] = {(uint16_t *)(ws + l.off_img[0]), (uint16_t *)(ws + l.off_img[1])};
    CUtensorMap mQ, mW, mPh[2], mImg[2];
    bool ok = make_map3(&mQ, Q, d, L, BH, 128) && make_map3(&mW, W, d, m, 1, m);
    for (int i = 0; ok && i < 2; ++i)
        ok = make_map3(&mPh[i], phi[i], m, L, BH, 128) && make_map3(&mImg[i], img[i], m, Np, BH, Np);
    if (!ok) return FAVOR_ERR_CUDA;
    if (launch_feature_offsets(W, m, d, c, st) != cudaSuccess) return FAVOR_ERR_CUDA;
    if (launch_reduce_image(state, 1, m, Np, img[0], img[1], BH, st) != cudaSuccess) return FAVOR_ERR_CUDA;
    GemmArgs aq = sp_args(L, m, d);
    aq.b_batched = 0;
    aq.ld_out = m;
    aq.out_hi = phi[0];
    aq.out_lo = phi[1];
    aq.colbias = c;
    if (launch_gemm_t<false, false, false, false, kEpiPhiQuery>(mQ, mQ, mW, mW, aq, m, BH, st) != cudaSuccess)
        return FAVOR_ERR_CUDA;
    GemmArgs ao = sp_args(L, Np, m);
    ao.ld_out = d;
    ao.out_f32 = out;
    ao.d = d;
    return cuda_status(
        launch_gemm_t<false, false, true, true, kEpiOut>(mPh[0], mPh[1], mImg[0], mImg[1], ao, Np, BH, st));
}

extern "C" favor_status favor_selftest_bounded_wait(unsigned int limit_us, void *stream) {
    if (limit_us == 0 || limit_us > 1000000u) return FAVOR_ERR_INVALID_ARG;
    return cuda_status(launch_wait_selftest(1000ull * limit_us, (cudaStream_t)stream));
}

// The no-allocation variant of the bidirectional forward (uses the definitions above).
#include "favor_static.cu"
