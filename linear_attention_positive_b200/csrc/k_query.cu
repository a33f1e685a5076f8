// Bidirectional state image and query-side output of the bf16 tensor-core path.
//
//   k_state_image : sums the per-run partial states in run order into the per-head state
//                   [S | z] = (K')^T [V | 1_L] (each run's per-feature stabilisers brought to one
//                   per-head reference), scales it by a power of two so that its largest
//                   magnitude lies in [2^14, 2^15), and writes it as fp16 in the layout the output
//                   MMA reads (the scale cancels between numerator and denominator).
//   k_query_out   : out = D^-1 (Q' S), D = diag(Q' z) ("Fast Attention Via Positive Orthogonal
//                   Random Features", codewithpapers.app/method/favor, the FA-part and its
//                   normaliser), with Q' = exp(Q W^T - rowmax) formed in TMEM and z riding along
//                   as one more column of the output MMA.
//
// State image of one head (fp16, B operand of the output MMA, K-major, 128-byte swizzle): for each
// value half nh (64 columns of d) and feature half h (128 features), two k-blocks of 64 features,
// each 80 rows x 128 bytes: row n < 64 holds S[., nh*64 + n], row 64 holds z, rows 65..79 are zero.
// Byte offset of (nh, h, kb, row n, 16-byte chunk p) = (((nh*H + h)*2 + kb)*80 + n)*128 + p*16,
// and chunk p holds features kb*64 + 8*(p ^ (n & 7)) + [0, 8) of the half.
//
// The causal path keeps the fp32 per-segment state blocks below (state_floats, state_image_offset).

#include <utility>

#include "common.cuh"

namespace favor {

__host__ __device__ inline size_t state_floats(int m, int d) { return (size_t)m * d + m + 4; }

__device__ __forceinline__ uint32_t state_image_offset(int r, int c, int m) {
    const int nh = c >> 6, cc = c & 63, kb = r >> 5, ch = (r & 31) >> 2, pos = r & 3;
    return (uint32_t)nh * (m * 64 * 4) + (uint32_t)kb * (64 * 128) + sw128_offset(cc, ch) + pos * 4;
}

constexpr int kImgRows = 80;                          // 64 value columns + z + 15 zero rows
constexpr uint32_t kImgKBlock = kImgRows * 128;       // bytes of one 64-feature k-block
constexpr uint32_t kImgHalf = 2 * kImgKBlock;         // bytes of one 128-feature half

// Bytes of one head's image (all value halves and feature halves).
__host__ __device__ inline size_t image_bytes(int m, int d) { return (size_t)(d / 64) * (m / 128) * kImgHalf; }

// ============================================================================ k_state_image

struct ImageParams {
    int m, d;
    Flat f;                  // partition of the key tiles (runs and their slots)
    const float *part;       // [slots][d+1][m]
    const float *part_D;     // [slots][m] per-run, per-feature stabilisers (log2 units)
    const float *part_amax;  // [slots][8]
    const float *part_Dmax;  // [slots][8]
    uint8_t *image;          // per head at image + bh * image_stride
    size_t image_stride;     // bytes
    float *key_ref;          // NULL, or [BH]: the head's reference stabiliser C (log2 units)
};

constexpr int kImageThreads = 128;

// 2^e for an integer-valued e (0 below 2^-126).
__device__ __forceinline__ float pow2i(float e) {
    const int i = (int)e;
    return i < -126 ? 0.f : __uint_as_float((uint32_t)(127 + i) << 23);
}

// One thread per 16-byte image chunk (8 features of one row). The head's runs are brought to one
// reference stabiliser C (the largest D over its runs and features): each run's feature row r is
// weighted by 2^(D_r - C), exactly, and summed in CTA order. The sums are scaled by 2^(15 - e),
// 2^e exceeding the bound sum_runs max_warp amax 2^(Dmax - C) on their magnitude, and rounded to
// fp16. Grid: (chunks / 128, heads).
__global__ void __launch_bounds__(kImageThreads) k_state_image(ImageParams p) {
    __shared__ float sC, sScale, sRed[kImageThreads / 32];
    pdl_launch_dependents();   // the query kernel may start its projections meanwhile
    pdl_wait_prerequisites();  // the key kernel's partial states are complete and visible
    const int bh = blockIdx.y;
    const int c_first = flat_first_cta(p.f, bh), c_last = flat_last_cta(p.f, bh);
    const int halves = p.m / 128, nhs = p.d / 64;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    // per-(run, warp) statistics, one per thread (a head spans at most a few runs)
    const int nstat = (c_last - c_first + 1) * 8;
    float dm = -INFINITY, am = 0.f;
    for (int i = threadIdx.x; i < nstat; i += kImageThreads) {
        if ((i & 7) < 4 * halves) {
            const size_t k = (size_t)(c_first + (i >> 3) + bh) * 8 + (i & 7);
            dm = fmaxf(dm, p.part_Dmax[k]);
        }
    }
    for (int o = 16; o > 0; o >>= 1) dm = fmaxf(dm, __shfl_xor_sync(0xffffffffu, dm, o));
    if (lane == 0) sRed[wid] = dm;
    __syncthreads();
    if (threadIdx.x == 0) {
        float C = sRed[0];
        for (int w = 1; w < kImageThreads / 32; ++w) C = fmaxf(C, sRed[w]);
        sC = C;
        // the backward's key features 2^(u log2e - C) stay below 2^19 (every run's D_r <= C)
        if (p.key_ref != nullptr && blockIdx.x == 0) p.key_ref[bh] = C;
    }
    __syncthreads();
    const float C = sC;
    for (int i = threadIdx.x; i < nstat; i += kImageThreads)
        if ((i & 7) < 4 * halves) {
            const size_t k = (size_t)(c_first + (i >> 3) + bh) * 8 + (i & 7);
            am = fmaxf(am, p.part_amax[k] * pow2i(p.part_Dmax[k] - C));  // per run the max over warps...
        }
    // ... summed over runs: every run's warps are taken by consecutive threads (8 per run), so the
    // bound is the sum over runs of the max over that run's 8 threads' values
    for (int o = 4; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    float bsum = (threadIdx.x & 7) == 0 ? am : 0.f;
    for (int o = 16; o > 0; o >>= 1) bsum += __shfl_xor_sync(0xffffffffu, bsum, o);
    __syncthreads();
    if (lane == 0) sRed[wid] = bsum;
    __syncthreads();
    if (threadIdx.x == 0) {
        float bound = 0.f;
        for (int w = 0; w < kImageThreads / 32; ++w) bound += sRed[w];
        // runs beyond the first kImageThreads / 8 (very short heads over many CTAs) were folded by
        // the strided loop into those threads' maxima: adding them per run keeps the bound valid
        if (nstat > kImageThreads) bound *= (float)((nstat + kImageThreads - 1) / kImageThreads);
        int ex = 0;
        frexpf(bound, &ex);  // bound < 2^ex
        sScale = bound > 0.f ? ldexpf(1.f, 15 - ex) : 1.f;
    }
    __syncthreads();
    const float scale = sScale;

    const int chunks = nhs * halves * 2 * kImgRows * 8;
    const int q = blockIdx.x * kImageThreads + threadIdx.x;
    if (q >= chunks) return;
    const int pch = q & 7, row = (q >> 3) % kImgRows, blk = (q >> 3) / kImgRows;  // blk = (nh*H + h)*2 + kb
    const int kb = blk & 1, h = (blk >> 1) % halves, nh = (blk >> 1) / halves;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (row <= 64) {
        const int col = row < 64 ? nh * 64 + row : p.d;
        const int r0 = h * 128 + kb * 64 + 8 * (pch ^ (row & 7));
        for (int c = c_first; c <= c_last; ++c) {
            const size_t slot = (size_t)(c + bh);
            const float4 *src = (const float4 *)(p.part + (slot * (p.d + 1) + col) * p.m + r0);
            const float4 *dd = (const float4 *)(p.part_D + slot * p.m + r0);
            const float4 a = src[0], b = src[1], da = dd[0], db = dd[1];
            v[0] = fmaf(a.x, pow2i(da.x - C), v[0]);
            v[1] = fmaf(a.y, pow2i(da.y - C), v[1]);
            v[2] = fmaf(a.z, pow2i(da.z - C), v[2]);
            v[3] = fmaf(a.w, pow2i(da.w - C), v[3]);
            v[4] = fmaf(b.x, pow2i(db.x - C), v[4]);
            v[5] = fmaf(b.y, pow2i(db.y - C), v[5]);
            v[6] = fmaf(b.z, pow2i(db.z - C), v[6]);
            v[7] = fmaf(b.w, pow2i(db.w - C), v[7]);
        }
    }
    uint4 u;
    u.x = pack_f16x2(v[0] * scale, v[1] * scale);
    u.y = pack_f16x2(v[2] * scale, v[3] * scale);
    u.z = pack_f16x2(v[4] * scale, v[5] * scale);
    u.w = pack_f16x2(v[6] * scale, v[7] * scale);
    *(uint4 *)(p.image + (size_t)bh * p.image_stride + ((size_t)blk * kImgRows + row) * 128 + pch * 16) = u;
}

// ============================================================================ k_query_out
//
// Persistent CTAs over a flat, head-major range of (head, value half, 128-query tile) items. The
// m features are split into 128-feature halves h, one per exponent warpgroup, each with its own
// TMEM buffers, so the halves never wait on each other's MMAs:
//   P_h = Q W_h^T (bf16 MMA into TMEM)
//   -> warpgroup h: row max of P_h, exchanged with the other half through shared memory, so both
//      use the row max over all m features, c; phi_h = 2^(P_h log2e - c) rounded to fp16, into TMEM
//   -> [O | den] = sum_h phi_h [S_h | z_h] (fp16 MMA, A from TMEM, N = 80: z rides along as one
//      more column of the state image)
//   -> epilogue warpgroup: out = O / den, staged in shared memory and written by TMA stores.
// Warp roles (16 warps): 0-3 epilogue, 4-7 / 8-11 exponentials of feature half 0 / 1, 12 TMA loads
// of Q and W, 13 MMA issue, 14 state image loads, 15 idle. Exponentials: per 32 columns, POLY go
// through the FMA-pipe polynomial and the rest through MUFU ex2, to balance the two pipes.
// TMEM columns: P_h [128h, +128), phi_h [256 + 64h, +64) (fp16 pairs), [O | den] [384, +80).

struct QueryParams {
    int L, d, m, BH, tiles_per_cta;
    const uint8_t *image;  // per head at image + bh * image_stride
    size_t image_stride;
};

constexpr int kQueryThreads = 512;
constexpr uint32_t kTmemPhi = 256, kTmemO = 384, kOCols = 80;

template <int D>
struct QueryCfg {
    static constexpr int KB = D / 64, NH = D / 64;
    static constexpr uint32_t Q_TILE = KB * kTile * 128;
    static constexpr int STAGES = D == 64 ? 3 : 2;
    static constexpr int OUT_BUFS = D == 64 ? 2 : 1;
    static constexpr uint32_t OUT_BUF = 4 * 2 * 32 * 128;  // 4 warps x two 32-column blocks x 32 rows
};

// One item's place in the CTA's range: head, value half, tile, and its (head, value half) group.
struct ItemInfo {
    int bh, nh, t, first_of_group, last_of_group, group;
};

template <int NH>
__device__ __forceinline__ ItemInfo item_info(int g, int f0, int f1, int nt) {
    ItemInfo it{};
    int group = 0;
    for (int bh = f0 / nt;; ++bh) {
        const int lo = max(f0, bh * nt) - bh * nt, hi = min(f1, (bh + 1) * nt) - bh * nt;
        const int n = hi - lo;
        if (g < NH * n) {
            it.bh = bh;
            it.nh = g / n;
            it.t = lo + g % n;
            it.first_of_group = (g % n) == 0;
            it.last_of_group = (g % n) == n - 1;
            it.group = group + it.nh;
            return it;
        }
        g -= NH * n;
        group += NH;
    }
}

// Row maximum of 128 values (four independent chains).
__device__ __forceinline__ float row_max128(const float (&v)[128]) {
    float a = -INFINITY, b = -INFINITY, c = -INFINITY, d = -INFINITY;
#pragma unroll
    for (int e = 0; e < 128; e += 8) {
        a = fmax3(a, v[e], v[e + 1]);
        b = fmax3(b, v[e + 2], v[e + 3]);
        c = fmax3(c, v[e + 4], v[e + 5]);
        d = fmax3(d, v[e + 6], v[e + 7]);
    }
    return fmaxf(fmaxf(a, b), fmaxf(c, d));
}

// phi = 2^(v log2e - cl) for a row of 128 logits, rounded to fp16 pairs. Per 32 columns the first
// 32 - POLY exponentials go to MUFU ex2, the last POLY to the FMA-pipe polynomial.
template <int POLY>
__device__ __forceinline__ void query_features(float (&v)[128], float cl, uint32_t (&hv)[64]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int e = c * 32; e < c * 32 + 32; e += 2) ffma2(v[e], v[e + 1], kLog2e, kLog2e, -cl, -cl, v[e], v[e + 1]);
#pragma unroll
        for (int e = c * 32; e < c * 32 + 32 - POLY; ++e) v[e] = ex2_approx(v[e]);
#pragma unroll
        for (int e = c * 32 + 32 - POLY; e < c * 32 + 32; e += 2) exp2_poly_pair(v[e], v[e + 1], v[e], v[e + 1]);
#pragma unroll
        for (int e = c * 32; e < c * 32 + 32; e += 2) hv[e >> 1] = pack_f16x2(v[e], v[e + 1]);
    }
}

template <int D, int POLY>
__global__ void __launch_bounds__(kQueryThreads, 1)
k_query_out(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapW,
            const __grid_constant__ CUtensorMap mapO, QueryParams p) {
    using C = QueryCfg<D>;
    constexpr int KB = C::KB, NH = C::NH, STAGES = C::STAGES;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int halves = p.m / 128;
    const uint32_t img_bytes = (uint32_t)halves * kImgHalf;
    uint8_t *sW = smem;                                              // KB x m x 128
    uint8_t *sImg = sW + (size_t)KB * p.m * 128;                     // halves x kImgHalf
    uint8_t *sQ = sImg + 2 * kImgHalf;                               // STAGES x Q_TILE
    uint8_t *sOut = sQ + (size_t)STAGES * C::Q_TILE;                 // OUT_BUFS x OUT_BUF
    float *sMax = (float *)(sOut + (size_t)C::OUT_BUFS * C::OUT_BUF);  // [2 parity][2 half][128]
    uint64_t *bars = (uint64_t *)(sMax + 512);
    uint64_t *full = bars, *empty = bars + STAGES;
    uint64_t *w_full = empty + STAGES, *img_full = w_full + 1, *img_empty = img_full + 1;
    uint64_t *p_full = img_empty + 1, *p_free = p_full + 1;
    uint64_t *xchg = p_free + 1;                                   // per item parity
    uint64_t *phi_full = xchg + 2, *phi_free = phi_full + 1;
    uint64_t *o_full = phi_free + 1, *o_empty = o_full + 1;
    uint64_t *drain = o_empty + 1;
    uint32_t *tmem_slot = (uint32_t *)(drain + 1);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nt = (p.L + kTile - 1) / kTile;
    const int total = p.BH * nt;
    const int f0 = blockIdx.x * p.tiles_per_cta;
    const int f1 = min(f0 + p.tiles_per_cta, total);
    const int n_items = NH * max(f1 - f0, 0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(w_full, 1);
        mbar_init(img_full, 1);
        mbar_init(img_empty, 1);
        mbar_init(p_full, 1);
        mbar_init(p_free, 128 * halves);
        mbar_init(&xchg[0], 128 * halves);
        mbar_init(&xchg[1], 128 * halves);
        mbar_init(phi_full, 128 * halves);
        mbar_init(phi_free, 1);
        mbar_init(o_full, 1);
        mbar_init(o_empty, 128);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 13) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 12) {
        regs_dec<56>();
        if (warp == 12 && n_items > 0) {
            // Q tiles (and W once).
            if (elect_one()) {
                prefetch_tensormap(&mapQ);
                prefetch_tensormap(&mapW);
                prefetch_tensormap(&mapO);
                mbar_arrive_expect_tx(w_full, KB * p.m * 128);
                for (int kb = 0; kb < KB; ++kb) tma_load_2d(sW + (size_t)kb * p.m * 128, &mapW, w_full, kb * 64, 0);
            }
            __syncwarp();
            int issued = 0;
            for (int g = 0; g < n_items; ++g) {
                const ItemInfo it = item_info<NH>(g, f0, f1, nt);
                const int s = g % STAGES;
                if (!mbar_wait_lazy(&empty[s], ((g / STAGES) & 1) ^ 1, abort_flag)) break;
                if (elect_one()) {
                    mbar_arrive_expect_tx(&full[s], C::Q_TILE);
                    for (int kb = 0; kb < KB; ++kb)
                        tma_load_3d(sQ + (size_t)s * C::Q_TILE + kb * kTile * 128, &mapQ, &full[s], kb * 64,
                                    it.t * kTile, it.bh);
                }
                __syncwarp();
                ++issued;
            }
            volatile int no_abort = 0;
            for (int i = max(issued - STAGES, 0); i < issued; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1, &no_abort);
            mbar_wait(w_full, 0, &no_abort);
        } else if (warp == 14 && n_items > 0) {
            // State image of each (head, value half) group, once the previous group's output
            // MMAs have finished with it. The image kernel (the launch before this one) must have
            // completed first: only this warp reads its output.
            pdl_wait_prerequisites();
            int groups = 0;
            for (int g = 0; g < n_items; ++g) {
                const ItemInfo it = item_info<NH>(g, f0, f1, nt);
                if (!it.first_of_group) continue;
                if (!mbar_wait_lazy(img_empty, (it.group & 1) ^ 1, abort_flag)) break;
                if (elect_one()) {
                    mbar_arrive_expect_tx(img_full, img_bytes);
                    const uint8_t *src = p.image + (size_t)it.bh * p.image_stride + (size_t)it.nh * img_bytes;
                    for (int h = 0; h < halves; ++h)
                        bulk_load(sImg + h * kImgHalf, src + h * kImgHalf, kImgHalf, img_full);
                }
                __syncwarp();
                ++groups;
            }
            volatile int no_abort = 0;
            if (groups > 0) mbar_wait(img_full, (groups - 1) & 1, &no_abort);
        } else if (warp == 13 && n_items > 0) {
            // MMA issue in a fixed order: the projection of item g+1 (both halves, N = m) as soon
            // as both halves' P have been read, then the output MMAs of item g once phi is in TMEM.
            const uint32_t idesc1 = make_idesc(kTile, p.m, kFmtBF16, 0, 0);
            const uint32_t idesc2 = make_idesc(kTile, kOCols, kFmtF16, 0, 0);
            const uint64_t dQ = make_sdesc(smem_u32(sQ), 16, 1024), dW = make_sdesc(smem_u32(sW), 16, 1024);
            const uint64_t dI = make_sdesc(smem_u32(sImg), 16, 1024);
            const uint32_t w_kb = (uint32_t)p.m * 128 / 16;  // W k-block stride, 16-byte units
            auto project = [&](int g) {
                const uint64_t a = dQ + (uint32_t)(g % STAGES) * (C::Q_TILE / 16);
                mma_ss_x4_w(tmem, a, dW, idesc1, 0u, 2, 2);
                if (KB == 2) mma_ss_x4_w(tmem, a + kTile * 128 / 16, dW + w_kb, idesc1, 1u, 2, 2);
                mma_commit_w(p_full);
            };
            bool ok = mbar_wait_all(w_full, 0, abort_flag) && mbar_wait_all(&full[0], 0, abort_flag);
            if (ok) {
                tc_fence_after();
                project(0);
                mma_commit_w(&empty[0]);
            }
            int bh = f0 / nt, nh = 0, t = f0 - bh * nt, group = 0;  // item g's place, advanced per item
            int run_end = min(f1, (bh + 1) * nt) - bh * nt;          // one past the last tile of this group
            int run_begin = t;
            for (int g = 0; ok && g < n_items; ++g) {
                const bool first = t == run_begin, last = t == run_end - 1;
                if (g + 1 < n_items) {
                    const int s1 = (g + 1) % STAGES;
                    if (!mbar_wait_all(&full[s1], ((g + 1) / STAGES) & 1, abort_flag)) break;
                    if (!mbar_wait_all(p_free, g & 1, abort_flag)) break;
                    tc_fence_after();
                    project(g + 1);
                    mma_commit_w(&empty[s1]);
                }
                if (first && !mbar_wait_all(img_full, group & 1, abort_flag)) break;
                if (g > 0 && !mbar_wait_all(o_empty, (g - 1) & 1, abort_flag)) break;
                if (!mbar_wait_all(phi_full, g & 1, abort_flag)) break;
                tc_fence_after();
                for (int h = 0; h < halves; ++h) {
                    const uint64_t b = dI + (uint32_t)h * (kImgHalf / 16);
                    mma_ts_x4_w(tmem + kTmemO, tmem + kTmemPhi + h * 64, b, idesc2, h > 0 ? 1u : 0u, 2);
                    mma_ts_x4_w(tmem + kTmemO, tmem + kTmemPhi + h * 64 + 32, b + kImgKBlock / 16, idesc2, 1u, 2);
                }
                mma_commit_w(phi_free);
                mma_commit_w(o_full);
                if (last) mma_commit_w(img_empty);
                // advance to item g + 1
                if (!last) {
                    ++t;
                } else if (nh + 1 < NH) {
                    ++nh;
                    ++group;
                    t = run_begin;
                } else {
                    ++bh;
                    nh = 0;
                    ++group;
                    run_begin = t = 0;
                    run_end = min(f1, (bh + 1) * nt) - bh * nt;
                }
            }
            mma_commit_w(drain);
            volatile int no_abort = 0;
            mbar_wait_all(drain, 0, &no_abort);
        }
    } else if (warp >= 4) {
        regs_inc<184>();
        // Warpgroup h: feature half h of every item (TMEM lane quarter = warp & 3).
        const int h = (warp - 4) >> 2, row = (warp & 3) * 32 + lane;
        if (h < halves) {
            const uint32_t lane_off = ((uint32_t)(warp & 3) * 32u) << 16;
            for (int g = 0; g < n_items; ++g) {
                if (!mbar_wait_all(p_full, g & 1, abort_flag)) break;
                tc_fence_after();
                float v[128];
                tmem_ld128(tmem + lane_off + h * 128, v);
                tc_fence_before();
                mbar_arrive(p_free);
                float rmax = row_max128(v);
                if (halves == 2) {
                    const int pb = g & 1;
                    sMax[(pb * 2 + h) * 128 + row] = rmax;
                    mbar_arrive(&xchg[pb]);
                    if (!mbar_wait_all(&xchg[pb], (g >> 1) & 1, abort_flag)) break;
                    rmax = fmaxf(rmax, sMax[(pb * 2 + (h ^ 1)) * 128 + row]);
                }
                uint32_t hv[64];
                query_features<POLY>(v, rmax * kLog2e, hv);
                if (g > 0 && !mbar_wait_all(phi_free, (g - 1) & 1, abort_flag)) break;
                tc_fence_after();
                tmem_st64(tmem + lane_off + kTmemPhi + h * 64, hv);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(phi_full);
            }
        }
    } else {
        regs_dec<88>();
        // Epilogue warpgroup: rows (warp)*32 + lane of every item.
        const uint32_t lane_off = ((uint32_t)warp * 32u) << 16;
        uint8_t *stage0 = sOut + warp * (2 * 32 * 128);
        for (int g = 0; g < n_items; ++g) {
            if (!mbar_wait_all(o_full, g & 1, abort_flag)) break;
            tc_fence_after();
            float o[64];
            tmem_ld64_nowait(tmem + lane_off + kTmemO, o);
            float den;
            asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=f"(den) : "r"(tmem + lane_off + kTmemO + 64));
            asm volatile("tcgen05.wait::ld.sync.aligned;" : FAVOR_RW32((&o[0])), FAVOR_RW32((&o[32])), "+f"(den)::"memory");
            tc_fence_before();
            mbar_arrive(o_empty);
            const float inv = 1.0f / den;
            uint8_t *stage = stage0 + (size_t)(g % C::OUT_BUFS) * C::OUT_BUF;
            if (lane == 0 && g >= C::OUT_BUFS) bulk_wait_group_read<C::OUT_BUFS - 1>();
            __syncwarp();
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                uint8_t *rowp = stage + cb * (32 * 128) + lane * 128;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const float *q = &o[cb * 32 + 4 * ch];
                    float4 w;
                    ffma2(q[0], q[1], inv, inv, 0.f, 0.f, w.x, w.y);
                    ffma2(q[2], q[3], inv, inv, 0.f, 0.f, w.z, w.w);
                    *(float4 *)(rowp + ((ch ^ (lane & 7)) << 4)) = w;
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                const ItemInfo it = item_info<NH>(g, f0, f1, nt);
                const int y = it.t * kTile + warp * 32;
                tma_store_3d(&mapO, stage, it.nh * 64, y, it.bh);
                tma_store_3d(&mapO, stage + 32 * 128, it.nh * 64 + 32, y, it.bh);
                bulk_commit_group();
            }
        }
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 13) tmem_dealloc(tmem, 512);
}

// ============================================================================ host launchers

template <int D>
static size_t query_smem(int m) {
    using C = QueryCfg<D>;
    return 1024 + (size_t)C::KB * m * 128 + 2 * kImgHalf + (size_t)C::STAGES * C::Q_TILE +
           (size_t)C::OUT_BUFS * C::OUT_BUF + 512 * 4 + 256;
}

// SM count of the current device (cached per device: the workspace layout and the persistent
// grids depend on it).
int num_sms() {
    constexpr int kMaxDev = 64;
    static int cached[kMaxDev] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) dev = 0;
    int n = cached[dev];
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return n;
}

// Launch with programmatic stream serialization: the kernel may be scheduled before the previous
// kernel on the stream completes; it waits (griddepcontrol.wait) before reading that kernel's output.
template <typename... KArgs, typename... Args>
static cudaError_t launch_after_previous(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                         Args &&...args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

cudaError_t launch_state_image(const ImageParams &p, int BH, cudaStream_t st) {
    const int chunks = (p.d / 64) * (p.m / 128) * 2 * kImgRows * 8;
    return launch_after_previous(k_state_image, dim3((chunks + kImageThreads - 1) / kImageThreads, BH),
                                 dim3(kImageThreads), 0, st, p);
}

// The register split of k_query_out (88 + 2 x 184 + 56 per warpgroup lane) adds up to the 128 per
// thread it is launched with; a build that launched with fewer would leave setmaxnreg waiting, so
// the launch is refused unless the kernel carries exactly 128.
template <typename Kern>
static bool query_regs_ok(Kern k) {
    cudaFuncAttributes a{};
    return cudaFuncGetAttributes(&a, k) == cudaSuccess && a.numRegs == 128;
}

template <int D, int POLY>
static cudaError_t launch_query_t(const CUtensorMap &mQ, const CUtensorMap &mW, const CUtensorMap &mO,
                                  const QueryParams &p, dim3 grid, cudaStream_t st) {
    static int checked = 0;  // 1 ok, -1 refused
    if (checked == 0) checked = query_regs_ok(k_query_out<D, POLY>) ? 1 : -1;
    if (checked < 0) return cudaErrorInvalidConfiguration;
    const size_t sm = query_smem<D>(p.m);
    cudaFuncSetAttribute(k_query_out<D, POLY>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    return launch_after_previous(k_query_out<D, POLY>, grid, dim3(kQueryThreads), sm, st, mQ, mW, mO, p);
}

// Persistent launch: at most one CTA per SM, each over a contiguous head-major range of tiles.
// poly_pct: share of exponentials taken by the FMA-pipe polynomial, rounded to 0, 25, 37.5 or 50
// percent (0, 8, 12 or 16 of every 32).
cudaError_t launch_query_out(const CUtensorMap &mQ, const CUtensorMap &mW, const CUtensorMap &mO, QueryParams p,
                             int poly_pct, cudaStream_t st) {
    const int total = p.BH * ((p.L + kTile - 1) / kTile);
    p.tiles_per_cta = (total + num_sms() - 1) / num_sms();
    const dim3 grid((total + p.tiles_per_cta - 1) / p.tiles_per_cta);
    const int poly = poly_pct < 13 ? 0 : poly_pct < 31 ? 8 : poly_pct < 44 ? 12 : 16;
    if (p.d == 64) {
        switch (poly) {
            case 0: return launch_query_t<64, 0>(mQ, mW, mO, p, grid, st);
            case 8: return launch_query_t<64, 8>(mQ, mW, mO, p, grid, st);
            case 12: return launch_query_t<64, 12>(mQ, mW, mO, p, grid, st);
            default: return launch_query_t<64, 16>(mQ, mW, mO, p, grid, st);
        }
    }
    switch (poly) {
        case 0: return launch_query_t<128, 0>(mQ, mW, mO, p, grid, st);
        case 8: return launch_query_t<128, 8>(mQ, mW, mO, p, grid, st);
        case 12: return launch_query_t<128, 12>(mQ, mW, mO, p, grid, st);
        default: return launch_query_t<128, 16>(mQ, mW, mO, p, grid, st);
    }
}

}  // namespace favor
