// Key side of the bidirectional bf16 tensor-core path for d = 64, on 128-token key tiles
// ("Fast Attention Via Positive Orthogonal Random Features", codewithpapers.app/method/favor: the
// FA-part needs (K')^T V and (K')^T 1_L).
//
//   k_key_partials_wide : per run, the partial state [S | z] = sum_j phi'(k_j) [v_j | 1] with
//                         phi'_r(k) = 2^(A - D_r) exp(u_r(k)), u_r(k) = w_r.k - |k|^2/2, D_r a
//                         per-feature stabiliser (log2 units) and A = 4. The output format is the
//                         one k_key_partials writes (same slots, same per-run maxima), so the state
//                         image kernel serves both.
//
// Why a second key kernel: on 64-token tiles each exponent warp spends most of a tile in fixed
// per-tile costs (barrier round trips, TMEM load latency, the stabiliser vote) rather than on the
// MUFU. Here a tile is 128 tokens and, except on a run's first tile, the projection is read once:
//   - P'_h^T = W_h K_tile^T + B'_j (M = 128 features of half h), issued as two N = 64 MMA groups,
//     one per 64-token half of the tile, so that each half of the P buffer is handed to the next
//     tile's projection as soon as the exponent warps are done with it. Each group is K = 64 of
//     W K^T plus one K = 16 extension step that adds the key's bias B'_j = B_j / log2e =
//     -|k_j|^2/2 + (A + b_t) ln 2: the converter warps write it as three bf16 parts (hi + mid + lo,
//     fp32's precision in sum) into the key row's extension, against three ones columns of W's;
//   - per 32-token chunk c: t = P' log2e - D_r (one paired FMA per two tokens), phi' = 2^t in fp16
//     stored to TMEM (16 packed columns) and z_r += 2^-b_t sum_j phi'; the next chunk's TMEM load is
//     in flight meanwhile. A warp vote on the chunk's fp32 sum of phi' (below the largest fp16
//     value no element can overflow) sends the rare chunk that may overflow to an out-of-line redo,
//     which re-reads its P columns and raises D_r where its largest t passes 15 (the causal use
//     votes on every chunk's largest t, which its head reference needs anyway);
//   - [S_h] += phi'_h V'_t (fp16 MMA, A from TMEM, B the converted V tile read MN-major, N = 64).
// z_r is kept in the exponent thread's registers instead of a ones column of the state MMA, which
// frees the TMEM columns the wider tile needs: per half P (128) + phi' (64) + S (64) = 256 columns.
//
// Stabiliser D_r (integer, per feature and run): on a run's first tile a separate pass over P finds
// the row's largest t and sets D_r so that it lands in (A+b-1, A+b]; on later tiles D_r is kept
// unless a chunk's largest t - D_r exceeds 15 (fp16 holds 2^t only below 2^16), in which case D_r
// is raised, the row's accumulated [S | z] and the tile's already stored phi' chunks are scaled by
// 2^-delta, and the chunk's exponentials are recomputed before they are stored. Typical inputs
// raise it rarely. V'_t = V_t 2^-b_t as in k_key_partials.
//
// Warp roles (16 warps): 0-3 the tile's largest |v| and b_t, convert V, write the key rows'
// extensions (thread j = token j of the tile); 4-7 / 8-11 exponentials of feature half 0 / 1 and
// the run-end write; 12 TMA; 13 / 15 MMA issue for half 0 / 1; 14 idle.

#include <type_traits>

#include "common.cuh"

namespace favor {

constexpr int kWideTile = 128;  // tokens per key tile of k_key_partials_wide

struct WideCfg {
    static constexpr int D = 64;
    static constexpr int STAGES = 4;
    static constexpr uint32_t TILE = kWideTile * 128;  // K or V tile: 128 rows of 64 bf16
    static constexpr uint32_t STAGE = 2 * TILE;        // K tile | V tile
    // key-row extension of a stage (interleaved, 128 rows x 32 bytes): B'_j in three bf16 parts
    static constexpr uint32_t KX = kWideTile * 32;
    // TMEM columns of half h (base h * 256): P [0, 128), phi' [128, 192), [S_h] [192, 256)
    static constexpr uint32_t T_P = 0, T_PHI = 128, T_S = 192, T_HALF = 256;
};

// Loads 16 consecutive 32-bit columns of this thread's TMEM lane and waits for them.
__device__ __forceinline__ void tmem_ld16u(uint32_t taddr, uint32_t (&h)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]), "=r"(h[4]), "=r"(h[5]), "=r"(h[6]), "=r"(h[7]), "=r"(h[8]),
          "=r"(h[9]), "=r"(h[10]), "=r"(h[11]), "=r"(h[12]), "=r"(h[13]), "=r"(h[14]), "=r"(h[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(h[0]), "+r"(h[1]), "+r"(h[2]), "+r"(h[3]), "+r"(h[4]), "+r"(h[5]), "+r"(h[6]), "+r"(h[7]),
                   "+r"(h[8]), "+r"(h[9]), "+r"(h[10]), "+r"(h[11]), "+r"(h[12]), "+r"(h[13]), "+r"(h[14]),
                   "+r"(h[15])::"memory");
}

// Largest value of a 32-token chunk.
__device__ __forceinline__ float chunk_vmax(const float (&v)[32]) {
    float a = -INFINITY, b = -INFINITY;
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
        a = fmax3(a, v[e], v[e + 1]);
        b = fmax3(b, v[e + 2], v[e + 3]);
    }
    return fmaxf(a, b);
}

// t = P' log2e - D for a 32-token chunk, in place (paired FMA-pipe instructions; P' carries the
// key's B_j through the projection's extension step); returns the chunk's largest t when MAX is set
// (else 0).
template <bool MAX>
__device__ __forceinline__ float chunk_shift(float (&v)[32], float D) {
    float a = -INFINITY, b = -INFINITY;
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
        ffma2(v[e], v[e + 1], kLog2e, kLog2e, -D, -D, v[e], v[e + 1]);
        ffma2(v[e + 2], v[e + 3], kLog2e, kLog2e, -D, -D, v[e + 2], v[e + 3]);
        if (MAX) {
            a = fmax3(a, v[e], v[e + 1]);
            b = fmax3(b, v[e + 2], v[e + 3]);
        }
    }
    return MAX ? fmaxf(a, b) : 0.f;
}

// Largest finite fp16 value: a chunk whose phi' sum stays below it has no element that overflows.
constexpr float kF16Max = 65504.f;

// phi' = 2^t for a 32-token chunk (t kept), rounded to fp16 pairs; returns the fp32 sum of phi'.
// The first 32 - POLY exponentials go to MUFU ex2, the last POLY to the FMA-pipe polynomial.
template <int POLY>
__device__ __forceinline__ float chunk_exp(const float (&t)[32], uint32_t (&hv)[16]) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        float e0, e1;
        if (e < 32 - POLY) {
            e0 = ex2_approx(t[e]);
            e1 = ex2_approx(t[e + 1]);
        } else {
            exp2_poly_pair(t[e], t[e + 1], e0, e1);
        }
        hv[e >> 1] = pack_f16x2(e0, e1);
        ffma2(e0, e1, 1.f, 1.f, s0, s1, s0, s1);
    }
    return s0 + s1;
}

// The two fp16 halves of a 32-bit word as fp32 (low half first).
__device__ __forceinline__ float2 unpack_f16x2(uint32_t h) {
    float lo, hi;
    asm("{\n\t.reg .b16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(h));
    return make_float2(lo, hi);
}

// Multiplies the fp16 pairs in 16 TMEM columns of this thread's lane by s (a power of two), in place.
__device__ __forceinline__ void tmem_scale_f16x16(uint32_t taddr, float s) {
    uint32_t h[16];
    tmem_ld16u(taddr, h);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float2 f = unpack_f16x2(h[i]);
        h[i] = pack_f16x2(f.x * s, f.y * s);
    }
    tmem_st16u(taddr, h);
    tmem_wait_st();
}

// Rare path of the exponent warps (warp-collective; out of line so that the common path's code
// stays compact): chunk c of the current tile, whose phi' may overflow fp16, is redone from its
// projection (tP: the chunk's P columns, still unreleased). Where the chunk's largest
// t passes 15, D_r is raised so that it lands at lim, and what already carries the old D_r -- the
// row's [S_h] (64 columns at tS), the tile's earlier phi' chunks, z and this tile's sum zs -- is
// scaled by 2^-delta. Stores the chunk's phi' and returns the updated scalars with its phi' sum.
struct KeyRaise {
    float Dr, z, zs, cs;
};
template <int POLY>
__device__ __noinline__ KeyRaise key_chunk_raise(uint32_t tP, uint32_t tPHI, uint32_t tS, int c, float Dr, float z,
                                                 float zs, float lim) {
    float v[32];
    tmem_ld32_nowait(tP, v);
    tmem_wait_ld32(v);
    const float cm = chunk_shift<true>(v, Dr);
    if (__any_sync(0xffffffffu, cm > 15.f)) {
        const float delta = cm > 15.f ? ceilf(cm - lim) : 0.f;
        const float sc = __uint_as_float((uint32_t)(127 - (int)delta) << 23);  // 2^-delta
        tmem_wait_st();
        tmem_scale_row(tS, WideCfg::D, sc);
        for (int cc = 0; cc < c; ++cc) tmem_scale_f16x16(tPHI + 16 * cc, sc);
        z *= sc;
        zs *= sc;
        Dr += delta;
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] -= delta;
    }
    uint32_t hv[16];
    const float cs = chunk_exp<POLY>(v, hv);
    tmem_st16u(tPHI + 16 * c, hv);
    return KeyRaise{Dr, z, zs, cs};
}

// Causal use of the kernel: the runs are the (head, segment) blocks of tps consecutive key tiles the
// causal scan works on (the last segment of a head may be shorter); each CTA takes whole segments.
struct WideSegParams {
    int n_split;       // segments per head
    int tps;           // tiles per segment
    int n_seg;         // BH * n_split
    int segs_per_cta;  // 0: bidirectional use (runs are the parts of heads inside CTA ranges)
    float *bias;       // [BH, L]: -|k_j|^2/2 per key (causal use), else NULL
    uint32_t *vmax;    // [n_seg]: the segment's largest |v| as bf16 bits (causal use), else NULL
};

// The key tiles of one CTA in order, with their run boundaries and run slot.
struct FlatWalk {  // bidirectional: tiles cta * T .. of the head-major flat order
    int bh, t, g, n, nt, cta;
    __device__ FlatWalk(const Flat &f, const WideSegParams &, int cta_) : nt(f.nt), cta(cta_) {
        const int fl = cta_ * f.T;
        n = max(min(fl + f.T, f.total) - fl, 0);
        bh = fl / f.nt;
        t = fl - bh * f.nt;
        g = 0;
    }
    __device__ bool first() const { return g == 0 || t == 0; }
    __device__ bool last() const { return g == n - 1 || t == nt - 1; }
    __device__ int slot() const { return cta + bh; }  // distinct for distinct (CTA, head) runs
    __device__ void next() {
        ++g;
        if (++t == nt) {
            t = 0;
            ++bh;
        }
    }
};
struct SegWalk {  // causal: whole segments of the CTA's range, one run each
    int sg, j, len, n, nt, n_split, tps, bh, t;
    __device__ int seg_len(int q) const { return min(tps, nt - (q % n_split) * tps); }
    __device__ SegWalk(const Flat &f, const WideSegParams &sp, int cta) : nt(f.nt), n_split(sp.n_split), tps(sp.tps) {
        const int s0 = cta * sp.segs_per_cta, s1 = min(s0 + sp.segs_per_cta, sp.n_seg);
        n = 0;
        for (int q = s0; q < s1; ++q) n += seg_len(q);
        sg = s0;
        j = 0;
        len = seg_len(sg);
        bh = sg / n_split;
        t = (sg - bh * n_split) * tps;
    }
    __device__ bool first() const { return j == 0; }
    __device__ bool last() const { return j == len - 1; }
    __device__ int slot() const { return sg; }
    __device__ void next() {
        ++t;
        if (++j == len) {
            ++sg;
            j = 0;
            len = seg_len(sg);
            bh = sg / n_split;
            t = (sg - bh * n_split) * tps;
        }
    }
};

template <int POLY, bool SEG>
__global__ void __launch_bounds__(kKeyThreads, 1)
k_key_partials_wide(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                    const __grid_constant__ CUtensorMap mapW, KeyStateParams2 p, WideSegParams sp) {
    using C = WideCfg;
    using Walk = typename std::conditional<SEG, SegWalk, FlatWalk>::type;
    constexpr int STAGES = C::STAGES, D = C::D;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int halves = p.m / 128;
    uint8_t *sW = smem;                                              // m rows of 128 B
    uint8_t *sStage = sW + (size_t)p.m * 128;                        // [STAGES] K tile | V tile
    uint8_t *sKx = sStage + (size_t)STAGES * C::STAGE;               // [STAGES] key-row extensions
    uint8_t *sWx = sKx + (size_t)STAGES * C::KX;                     // m feature rows x 32 B: 1, 1, 1, 0...
    int *sShift = (int *)(sWx + (size_t)p.m * 32);                   // [STAGES] b_t; [8, 16) converter scratch
    uint64_t *bars = (uint64_t *)(sShift + 16);
    uint64_t *full = bars, *empty = full + STAGES, *conv_full = empty + STAGES;
    // per feature half h: p_full / p_free [2h + q] (P columns of token half q), phi_full / phi_free
    // (the phi' buffer), acc_full / acc_empty ([S_h] at a run's end), drain (the half's MMAs at exit)
    uint64_t *w_full = conv_full + STAGES, *p_full = w_full + 1, *p_free = p_full + 4, *phi_full = p_free + 4;
    uint64_t *phi_free = phi_full + 2, *acc_full = phi_free + 2, *acc_empty = acc_full + 2, *drain = acc_empty + 2;
    uint32_t *tmem_slot = (uint32_t *)(drain + 2);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    pdl_launch_dependents();  // the state image kernel may stage its launch meanwhile
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = Walk(p.f, sp, blockIdx.x).n;  // key tiles of this CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], halves);  // one MMA commit per feature half
            mbar_init(&conv_full[s], 128);
        }
        mbar_init(w_full, 1);
        for (int q = 0; q < 4; ++q) {
            mbar_init(&p_full[q], 1);
            mbar_init(&p_free[q], 128);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&phi_full[h], 128);
            mbar_init(&phi_free[h], 1);
            mbar_init(&acc_full[h], 1);
            mbar_init(&acc_empty[h], 128);
            mbar_init(&drain[h], 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 13) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    // Projection extension (one K = 16 step, interleaved layout: row r's 16-byte core-matrix row at
    // (r / 8) 256 + (k / 8) 128 + (r % 8) 16): W's rows get three ones columns, every key row's
    // second core matrix is zero (the first is written per tile by the converter warps).
    for (int i = threadIdx.x; i < p.m * 2; i += kKeyThreads) {
        const int r = i >> 1, kc = i & 1;
        *(uint4 *)(sWx + (r >> 3) * 256 + kc * 128 + (r & 7) * 16) =
            kc == 0 ? make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
    }
    for (int i = threadIdx.x; i < STAGES * kWideTile; i += kKeyThreads) {
        const int st = i / kWideTile, r = i % kWideTile;
        *(uint4 *)(sKx + st * C::KX + (r >> 3) * 256 + 128 + (r & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 12) {
        regs_dec<88>();
        if (warp == 12 && n > 0) {
            if (elect_one()) {
                prefetch_tensormap(&mapK);
                prefetch_tensormap(&mapV);
                prefetch_tensormap(&mapW);
                mbar_arrive_expect_tx(w_full, p.m * 128);
                tma_load_2d(sW, &mapW, w_full, 0, 0);
            }
            __syncwarp();
            int issued = 0;
            Walk wk(p.f, sp, blockIdx.x);
            for (int g = 0; g < n; ++g, wk.next()) {
                const int s = g % STAGES;
                // the later stages' first loads wait until tile 0 has landed: at launch every CTA asks
                // for its first tile alone, so that it arrives sooner
                if (g == 1 && !mbar_wait_all(&full[0], 0, abort_flag)) break;
                if (!mbar_wait_lazy(&empty[s], ((g / STAGES) & 1) ^ 1, abort_flag)) break;
                if (elect_one()) {
                    uint8_t *st = sStage + (size_t)s * C::STAGE;
                    mbar_arrive_expect_tx(&full[s], 2 * C::TILE);
                    tma_load_3d(st, &mapK, &full[s], 0, wk.t * kWideTile, wk.bh);
                    tma_load_3d(st + C::TILE, &mapV, &full[s], 0, wk.t * kWideTile, wk.bh);
                }
                __syncwarp();
                ++issued;
            }
            volatile int no_abort = 0;
            for (int i = max(issued - STAGES, 0); i < issued; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1, &no_abort);
            mbar_wait(w_full, 0, &no_abort);
        } else if ((warp == 13 || (warp == 15 && halves == 2)) && n > 0) {
            // MMA issue for feature half h by the whole converged warp (predicated issue forms): per
            // tile g, the projection of tile g + 1's first 64 tokens once the exponent warps are done
            // with P(g)'s columns 0-63, the state MMA of tile g once its V tile is converted and
            // phi'(g) is in TMEM, then the projection of tile g + 1's last 64 tokens.
            const int h = warp == 13 ? 0 : 1;
            const uint32_t tH = tmem + (uint32_t)h * C::T_HALF;
            const uint32_t idesc_p = make_idesc(128, kWideTile / 2, kFmtBF16, 0, 0);
            const uint32_t idesc_s = make_idesc(128, D, kFmtF16, 0, 1);
            const uint64_t dW = make_sdesc(smem_u32(sW) + (uint32_t)h * 128 * 128, 16, 1024);
            const uint64_t dK = make_sdesc(smem_u32(sStage), 16, 1024);
            const uint64_t dV = make_sdesc(smem_u32(sStage) + C::TILE, C::TILE, 1024);
            // token half q of tile g (K rows 64q.., 64 swizzled rows = 8 KB) into P columns 64q..
            // plus the extension step: B'_j of token half q against W's ones columns
            const uint64_t dWx = make_sdesc_interleaved(smem_u32(sWx) + (uint32_t)h * 4096, 128, 256);
            const uint64_t dKx = make_sdesc_interleaved(smem_u32(sKx), 128, 256);
            auto project = [&](int g, int q) {
                const uint64_t kd = dK + (uint32_t)(g % STAGES) * (C::STAGE / 16) + (uint32_t)q * (8192 / 16);
                mma_ss_x4_w(tH + C::T_P + 64 * q, dW, kd, idesc_p, 0u, 2, 2);
                const uint64_t xd = dKx + (uint32_t)(g % STAGES) * (C::KX / 16) + (uint32_t)q * (2048 / 16);
                mma_f16_ss_w(tH + C::T_P + 64 * q, dWx, xd, idesc_p, 1u);
                mma_commit_w(&p_full[2 * h + q]);
            };
            // a projection reads the tile's key rows (TMA) and their extension (converter warps)
            bool ok = mbar_wait_all(w_full, 0, abort_flag) && mbar_wait_all(&full[0], 0, abort_flag) &&
                      mbar_wait_all(&conv_full[0], 0, abort_flag);
            tc_fence_after();
            if (ok) {
                project(0, 0);
                project(0, 1);
            }
            int runs = 0;
            Walk wk(p.f, sp, blockIdx.x);
            for (int g = 0; ok && g < n; ++g, wk.next()) {
                const int s = g % STAGES;
                const bool first = wk.first(), last = wk.last();
                if (g + 1 < n) {
                    ok = mbar_wait_all(&full[(g + 1) % STAGES], ((g + 1) / STAGES) & 1, abort_flag) &&
                         mbar_wait_all(&conv_full[(g + 1) % STAGES], ((g + 1) / STAGES) & 1, abort_flag) &&
                         mbar_wait_all(&p_free[2 * h], g & 1, abort_flag);
                    tc_fence_after();
                    if (!ok) break;
                    project(g + 1, 0);
                }
                ok = mbar_wait_all(&conv_full[s], (g / STAGES) & 1, abort_flag);
                if (ok && first && runs > 0) ok = mbar_wait_all(&acc_empty[h], (runs - 1) & 1, abort_flag);
                if (ok) ok = mbar_wait_all(&phi_full[h], g & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint64_t vd = dV + (uint32_t)s * (C::STAGE / 16);
                mma_ts_x4_w(tH + C::T_S, tH + C::T_PHI, vd, idesc_s, first ? 0u : 1u, 2048 / 16);
                mma_ts_x4_w(tH + C::T_S, tH + C::T_PHI + 32, vd + 8192 / 16, idesc_s, 1u, 2048 / 16);
                mma_commit_w(&phi_free[h]);
                if (last) {
                    mma_commit_w(&acc_full[h]);
                    ++runs;
                }
                mma_commit_w(&empty[s]);
                if (g + 1 < n) {
                    ok = mbar_wait_all(&p_free[2 * h + 1], g & 1, abort_flag);
                    tc_fence_after();
                    if (!ok) break;
                    project(g + 1, 1);
                }
            }
            mma_commit_w(&drain[h]);
            volatile int no_abort = 0;
            mbar_wait_all(&drain[h], 0, &no_abort);
        }
    } else if (warp >= 4) {
        regs_inc<160>();
        const int h = (warp - 4) >> 2, row = (warp & 3) * 32 + lane;
        if (h < halves && n > 0) {
            const uint32_t lane_off = ((uint32_t)(warp & 3) * 32u) << 16;
            const uint32_t tH = tmem + lane_off + (uint32_t)h * C::T_HALF;
            const uint32_t tP = tH + C::T_P, tPHI = tH + C::T_PHI, tS = tH + C::T_S;
            int runs = 0;
            float Dr = 0.f;  // this feature's stabiliser D_r in the current run
            float z = 0.f;   // this feature's normaliser entry z_r of the current run (2^-b_t scale)
            float umax = -INFINITY;  // the run's largest t - b_t = u log2e + A (causal use)
            Walk wk(p.f, sp, blockIdx.x);
            float va[32], vb[32];
            for (int g = 0; g < n; ++g, wk.next()) {
                const int s = g % STAGES;
                const bool first = wk.first(), last = wk.last();
                if (!mbar_wait_all(&p_full[2 * h], g & 1, abort_flag) ||
                    !mbar_wait_all(&conv_full[s], (g / STAGES) & 1, abort_flag))
                    break;
                tc_fence_after();
                const int bt = sShift[s];
                const float lim = kKeyFeatureShift + (float)bt;  // target for a run's largest t
                if (first) {
                    // a run's first tile: D_r from the row's largest t over the whole tile
                    tmem_ld32_nowait(tP, va);
                    tmem_wait_ld32(va);
                    tmem_ld32_nowait(tP + 32, vb);
                    float pm = chunk_vmax(va);
                    tmem_wait_ld32(vb);
                    if (!mbar_wait_all(&p_full[2 * h + 1], g & 1, abort_flag)) break;
                    tc_fence_after();
                    tmem_ld32_nowait(tP + 64, va);
                    pm = fmaxf(pm, chunk_vmax(vb));
                    tmem_wait_ld32(va);
                    tmem_ld32_nowait(tP + 96, vb);
                    pm = fmaxf(pm, chunk_vmax(va));
                    tmem_wait_ld32(vb);
                    pm = fmaxf(pm, chunk_vmax(vb));
                    const float tm = pm * kLog2e;  // the rounding of t = P' log2e is monotone
                    Dr = ceilf(tm - lim);
                    z = 0.f;
                    umax = tm - (float)bt;
                }
                float zs = 0.f;  // this tile's sum of phi'
                // One 32-token chunk: t and phi'. On a later tile of the run, a chunk that may overflow
                // fp16 is redone out of line (key_chunk_raise: D_r raised where a largest t passes 15).
                // The vote takes the chunk's fp32 sum of phi' (below the largest fp16 value no element
                // can overflow), or in causal use its largest t, which the head reference needs anyway.
                // phi'(g) overwrites phi'(g - 1), so before the first store the state MMA of tile g - 1
                // must have read it (which also makes [S] safe to rescale). `pend` is the buffer whose
                // TMEM load is in flight: the rare path completes it before the call.
                auto chunk = [&](float(&v)[32], float(&pend)[32], bool has_pend, int c) -> bool {
                    const float cm = SEG ? chunk_shift<true>(v, Dr) : chunk_shift<false>(v, Dr);
                    if (SEG && !first) umax = fmaxf(umax, cm + Dr - (float)bt);
                    uint32_t hv[16];
                    const float cs = chunk_exp<POLY>(v, hv);
                    if (c == 0) {
                        if (g > 0 && !mbar_wait_all(&phi_free[h], (g - 1) & 1, abort_flag)) return false;
                        tc_fence_after();
                    }
                    if (!first && __any_sync(0xffffffffu, SEG ? cm > 15.f : cs >= kF16Max)) {
                        if (has_pend) tmem_wait_ld32(pend);
                        const KeyRaise r = key_chunk_raise<POLY>(tP + 32 * c, tPHI, tS, c, Dr, z, zs, lim);
                        Dr = r.Dr;
                        z = r.z;
                        zs = r.zs + r.cs;
                    } else {
                        zs += cs;
                        tmem_st16u(tPHI + 16 * c, hv);
                    }
                    return true;
                };
                // P columns 0-63 (token half 0) stay readable until chunks 0 and 1 are done (a redo
                // reads them again), columns 64-127 until chunk 3 is done; each half is then handed to
                // the projection of tile g + 1.
                tmem_ld32_nowait(tP, va);
                tmem_wait_ld32(va);
                tmem_ld32_nowait(tP + 32, vb);
                if (!chunk(va, vb, true, 0)) break;
                tmem_wait_ld32(vb);
                if (!first) {
                    if (!mbar_wait_all(&p_full[2 * h + 1], g & 1, abort_flag)) break;
                    tc_fence_after();
                }
                tmem_ld32_nowait(tP + 64, va);
                chunk(vb, va, true, 1);
                tc_fence_before();
                mbar_arrive(&p_free[2 * h]);
                tmem_wait_ld32(va);
                tmem_ld32_nowait(tP + 96, vb);
                chunk(va, vb, true, 2);
                tmem_wait_ld32(vb);
                chunk(vb, va, false, 3);
                tc_fence_before();
                mbar_arrive(&p_free[2 * h + 1]);
                z = fmaf(zs, __uint_as_float((uint32_t)(127 - bt) << 23), z);  // z_r += 2^-b_t sum_j phi'
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&phi_full[h]);
                if (last) {
                    if (!mbar_wait_all(&acc_full[h], runs & 1, abort_flag)) break;
                    tc_fence_after();
                    const size_t rs = (size_t)wk.slot();
                    float *dst = p.part + rs * (D + 1) * p.m + h * 128 + row;
                    float amax = fabsf(z);
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        tmem_ld32(tS + c0, va);
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            dst[(size_t)(c0 + c) * p.m] = va[c];
                            amax = fmaxf(amax, fabsf(va[c]));
                        }
                    }
                    tc_fence_before();
                    mbar_arrive(&acc_empty[h]);
                    dst[(size_t)D * p.m] = z;
                    p.part_D[rs * p.m + h * 128 + row] = Dr;
                    float dmax = SEG ? umax : Dr;
                    for (int o = 16; o > 0; o >>= 1) {
                        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                        dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, o));
                    }
                    if (lane == 0) {
                        p.part_amax[rs * 8 + h * 4 + (warp & 3)] = amax;
                        p.part_Dmax[rs * 8 + h * 4 + (warp & 3)] = dmax;
                    }
                    ++runs;
                }
            }
        }
    } else {
        regs_dec<88>();
        // Converter warpgroup: thread j handles token j of each tile (its |k_j|^2 and extension) and 8 of
        // the V tile's 16-byte chunks. The largest |v| of the tile (bf16 magnitudes compared as
        // integers, reduced over the warpgroup) gives b_t; the chunks are then rewritten as fp16
        // V' = V 2^-b_t. In causal use thread 0 also records each segment's largest |v|.
        const int j = threadIdx.x;
        uint32_t *sRed = (uint32_t *)(sShift + 8);  // [2 tile parities][4 warps]
        uint32_t run_mx = 0;
        Walk wk(p.f, sp, blockIdx.x);
        for (int g = 0; g < n; ++g, wk.next()) {
            const int s = g % STAGES, t = wk.t;
            // the first tile is on every CTA's critical path: poll it without sleeping
            const bool ok = g == 0 ? mbar_wait_all(&full[0], 0, abort_flag)
                                   : mbar_wait_lazy(&full[s], (g / STAGES) & 1, abort_flag);
            if (!ok) break;
            uint8_t *st = sStage + (size_t)s * C::STAGE;
            uint4 vw[C::TILE / 16 / 128];
            uint32_t mx = 0;
#pragma unroll
            for (int i = 0; i < (int)(C::TILE / 16 / 128); ++i) {
                vw[i] = *(const uint4 *)(st + C::TILE + (size_t)(j + 128 * i) * 16);
                mx = __vmaxu2(mx, vw[i].x & 0x7FFF7FFFu);
                mx = __vmaxu2(mx, vw[i].y & 0x7FFF7FFFu);
                mx = __vmaxu2(mx, vw[i].z & 0x7FFF7FFFu);
                mx = __vmaxu2(mx, vw[i].w & 0x7FFF7FFFu);
            }
            mx = max(mx & 0xFFFFu, mx >> 16);
            for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if ((j & 31) == 0) sRed[(g & 1) * 4 + (j >> 5)] = mx;
            named_bar_sync(1, 128);
            mx = max(max(sRed[(g & 1) * 4], sRed[(g & 1) * 4 + 1]), max(sRed[(g & 1) * 4 + 2], sRed[(g & 1) * 4 + 3]));
            const int e = (int)(mx >> 7) - 127;  // exponent of the largest |v| (-127 for an all-zero tile)
            const int b = min(max(e - 7, -8), 7);
            if (j == 0) {
                sShift[s] = b;
                // V' = V 2^-b_t is an fp16 operand: from 2^23 on (and for inf / nan) it would overflow
                if (mx >= 0x4B00u) record_status(FAVOR_ERR_UNSUPPORTED);
                if (SEG) {
                    run_mx = max(run_mx, mx);
                    if (wk.last()) {
                        sp.vmax[wk.slot()] = run_mx;
                        run_mx = 0;
                    }
                }
            }
            const float scale = __uint_as_float((uint32_t)(127 - b) << 23);  // 2^-b
#pragma unroll
            for (int i = 0; i < (int)(C::TILE / 16 / 128); ++i) {
                uint32_t u[4] = {vw[i].x, vw[i].y, vw[i].z, vw[i].w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float lo, hi;
                    ffma2(__uint_as_float(u[k] << 16), __uint_as_float(u[k] & 0xFFFF0000u), scale, scale, 0.f, 0.f, lo, hi);
                    u[k] = pack_f16x2(lo, hi);
                }
                *(uint4 *)(st + C::TILE + (size_t)(j + 128 * i) * 16) = make_uint4(u[0], u[1], u[2], u[3]);
            }
            const bool valid = t * kWideTile + j < p.L;
            const float k2 = key_sq_norm<1, kWideTile>(st, j);
            // B'_j = B_j / log2e = -|k_j|^2 / 2 + (A + b_t) ln 2 as three bf16 parts (hi, mid, lo: their
            // sum carries fp32's precision) in key row j's extension; a key past L gets -inf
            uint4 xb = make_uint4(0xFF80u, 0u, 0u, 0u);
            if (valid) {
                const float Bp = fmaf(-0.5f, k2, (kKeyFeatureShift + (float)b) * kLn2);
                const uint32_t hi = bf16_bits_rn(Bp);
                const float r1 = Bp - __uint_as_float(hi << 16);
                const uint32_t mid = bf16_bits_rn(r1);
                const uint32_t lo = bf16_bits_rn(r1 - __uint_as_float(mid << 16));
                xb = make_uint4(hi | (mid << 16), lo, 0u, 0u);
            }
            *(uint4 *)(sKx + s * C::KX + (j >> 3) * 256 + (j & 7) * 16) = xb;
            if (SEG && valid) sp.bias[(size_t)wk.bh * p.L + t * kWideTile + j] = -0.5f * k2;
            fence_async_smem();
            mbar_arrive(&conv_full[s]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 13) tmem_dealloc(tmem, 512);
}

// ============================================================================ host launchers

static size_t key_wide_smem(int m) {
    using C = WideCfg;
    return 1024 + (size_t)m * 128 + (size_t)C::STAGES * (C::STAGE + C::KX) + (size_t)m * 32 + 64 + 512;
}

// The register split (88 + 2 x 160 + 88 per warpgroup lane) fits the 128 per thread the kernel is
// launched with; the launch is refused unless the kernel carries exactly 128.
template <int POLY, bool SEG>
static cudaError_t launch_key_wide_t(const CUtensorMap &mK, const CUtensorMap &mV, const CUtensorMap &mW,
                                     const KeyStateParams2 &p, const WideSegParams &sp, int n_cta, cudaStream_t st) {
    static int checked = 0;
    if (checked == 0) {
        cudaFuncAttributes a{};
        checked = (cudaFuncGetAttributes(&a, k_key_partials_wide<POLY, SEG>) == cudaSuccess && a.numRegs == 128) ? 1 : -1;
    }
    if (checked < 0) return cudaErrorInvalidConfiguration;
    const size_t sm = key_wide_smem(p.m);
    cudaFuncSetAttribute(k_key_partials_wide<POLY, SEG>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_key_partials_wide<POLY, SEG><<<n_cta, kKeyThreads, sm, st>>>(mK, mV, mW, p, sp);
    return cudaGetLastError();
}

template <bool SEG>
static cudaError_t launch_key_wide_poly(const CUtensorMap &mK, const CUtensorMap &mV, const CUtensorMap &mW,
                                        const KeyStateParams2 &p, const WideSegParams &sp, int n_cta, int poly_pct,
                                        cudaStream_t st) {
    const int poly = poly_pct < 13 ? 0 : poly_pct < 31 ? 8 : poly_pct < 44 ? 12 : 16;
    switch (poly) {
        case 0: return launch_key_wide_t<0, SEG>(mK, mV, mW, p, sp, n_cta, st);
        case 8: return launch_key_wide_t<8, SEG>(mK, mV, mW, p, sp, n_cta, st);
        case 12: return launch_key_wide_t<12, SEG>(mK, mV, mW, p, sp, n_cta, st);
        default: return launch_key_wide_t<16, SEG>(mK, mV, mW, p, sp, n_cta, st);
    }
}

// Bidirectional use, d = 64: K and V maps with 128-row boxes, p.f built on 128-token tiles.
cudaError_t launch_key_partials_wide(const CUtensorMap &mK, const CUtensorMap &mV, const CUtensorMap &mW,
                                     const KeyStateParams2 &p, int poly_pct, cudaStream_t st) {
    const WideSegParams none{0, 0, 0, 0, nullptr, nullptr};
    return launch_key_wide_poly<false>(mK, mV, mW, p, none, p.f.n_cta, poly_pct, st);
}

// Causal use, d = 64: one run per (head, segment of sp.tps tiles), each CTA taking sp.segs_per_cta
// whole segments; slot = segment index (head-major). p.part_Dmax receives, per (slot, half, warp),
// the run's largest u log2e + A instead of its largest D_r, and sp.bias the per-key -|k|^2/2.
cudaError_t launch_key_segments(const CUtensorMap &mK, const CUtensorMap &mV, const CUtensorMap &mW,
                                const KeyStateParams2 &p, const WideSegParams &sp, int poly_pct, cudaStream_t st) {
    const int n_cta = (sp.n_seg + sp.segs_per_cta - 1) / sp.segs_per_cta;
    return launch_key_wide_poly<true>(mK, mV, mW, p, sp, n_cta, poly_pct, st);
}

// ============================================================================ k_segment_scan
//
// Causal use: the exclusive prefix over a head's segments of the state the chunked scan starts
// each segment from, at the head's key reference. Segment sg of k_key_partials_wide holds
// [S'_r | z'_r] = 2^(A - D_r) sum_j e^(u_r(k_j)) [v_j | 1] (A the key shift 4, D_r its per-feature
// stabiliser); with C = max over the head's keys and features of u (nats), taken from the segments'
// largest u log2e + A, the prefix of segment sp is 2^8 sum_{sg < sp} 2^(D_r - A - C log2e) [S' | z']
// = 2^8 sum_j e^(u_r(k_j) - C) [v_j | 1] over the keys before the segment: the form k_causal_chunk
// reads (keys 2^8 below fp16's limit under C). One thread per element (value column c, feature r),
// feature-minor like the partial states, so reads and writes are coalesced; eight segments' loads
// in flight.

struct SegScanParams {
    int m, n_split, halves;
    const float *part;       // [n_seg][65][m]
    const float *part_D;     // [n_seg][m]
    const float *part_umax;  // [n_seg][8]: per (half, warp) largest u log2e + A
    float *seg_S;            // [BH][n_split][64][m]
    float *seg_z;            // [BH][n_split][m]
    float *head_max;         // [BH]: C (nats)
    float *key_ref;          // NULL or [BH]: C log2e
};

__global__ void __launch_bounds__(256) k_segment_scan(SegScanParams p) {
    constexpr int D = 64, NC = D + 1;
    __shared__ float sRed[8];
    const int bh = blockIdx.y;
    pdl_wait_prerequisites();  // the key kernel's segments are complete and visible
    // the head's reference: the largest u log2e + A over its segments
    float mx = -INFINITY;
    for (int i = threadIdx.x; i < p.n_split * 8; i += 256)
        if ((i & 7) < 4 * p.halves) mx = fmaxf(mx, p.part_umax[((size_t)bh * p.n_split + (i >> 3)) * 8 + (i & 7)]);
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) sRed[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = sRed[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) mx = fmaxf(mx, sRed[i]);
    const float kref = mx - kKeyFeatureShift;  // C log2e
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        p.head_max[bh] = kref / kLog2e;
        if (p.key_ref) p.key_ref[bh] = kref;
    }
    const size_t i = (size_t)blockIdx.x * 256 + threadIdx.x;
    if (i >= (size_t)NC * p.m) return;
    const int c = (int)(i / p.m), r = (int)(i - (size_t)c * p.m);
    const size_t seg0 = (size_t)bh * p.n_split;
    const float *src = p.part + seg0 * NC * p.m + i;
    const float *dsrc = p.part_D + seg0 * p.m + r;
    const size_t sstride = (size_t)NC * p.m;
    float *dst;
    size_t dstride;
    if (c < D) {
        dst = p.seg_S + seg0 * D * p.m + (size_t)c * p.m + r;
        dstride = (size_t)D * p.m;
    } else {
        dst = p.seg_z + seg0 * p.m + r;
        dstride = p.m;
    }
    const float off = kKeyFeatureShift + kref;
    float run = 0.f;
    int sp = 0;
    for (; sp + 8 <= p.n_split; sp += 8) {
        float a[8], dd[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            a[k] = src[(size_t)(sp + k) * sstride];
            dd[k] = dsrc[(size_t)(sp + k) * p.m];
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            dst[(size_t)(sp + k) * dstride] = run * 256.f;  // exclusive prefix, times 2^8
            run = fmaf(exp2f(dd[k] - off), a[k], run);
        }
    }
    for (; sp < p.n_split; ++sp) {
        dst[(size_t)sp * dstride] = run * 256.f;
        run = fmaf(exp2f(dsrc[(size_t)sp * p.m] - off), src[(size_t)sp * sstride], run);
    }
}

cudaError_t launch_segment_scan(const SegScanParams &p, int BH, cudaStream_t st) {
    return launch_after_previous(k_segment_scan, dim3((65 * p.m + 255) / 256, BH), dim3(256), 0, st, p);
}

}  // namespace favor
