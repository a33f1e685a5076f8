// Key side of the bidirectional bf16 tensor-core path for d = 128 on 64-token key tiles ("Fast
// Attention Via Positive Orthogonal Random Features", codewithpapers.app/method/favor: the FA-part
// needs (K')^T V and (K')^T 1_L). d = 64 runs on k_key_partials_wide (k_keys_wide.cu), which also
// uses this file's shared pieces (Flat, key_sq_norm, KeyStateParams2, tmem_scale_row).
//
//   k_key_partials : per run, the partial state [S | z] = sum_j phi'(k_j) [v_j | 1] with
//                    phi'_r(k) = 2^(A - D_r) exp(u_r(k)), u_r(k) = w_r.k - |k|^2/2, where D_r is a
//                    per-feature stabiliser kept by the run (log2 units) and A = 4. The image
//                    kernel brings every run and feature to one per-(batch, head) reference
//                    before the state is used, so the stabilisers cancel in D^-1.
//
// Work split: the BH * ceil(L/64) key tiles, head-major, are cut into contiguous ranges of T
// tiles, one per persistent CTA.
// A run is the part of one head inside one CTA's range; run
// (CTA c, head bh) owns slot c + bh of the per-run outputs (runs are ordered by both c and bh, so
// c + bh is distinct for distinct runs). A head's runs are the CTAs first_cta(bh)..last_cta(bh).

#include "common.cuh"

namespace favor {

// Flat partition of the key (or query) tiles over persistent CTAs.
struct Flat {
    int nt;     // tiles per head
    int total;  // BH * nt
    int T;      // tiles per CTA
    int n_cta;  // CTAs launched
};

inline Flat make_flat(int BH, int L, int n_sms, int tile = kTile) {
    Flat f;
    f.nt = (L + tile - 1) / tile;
    f.total = BH * f.nt;
    f.T = (f.total + n_sms - 1) / n_sms;
    f.n_cta = (f.total + f.T - 1) / f.T;
    return f;
}
__host__ __device__ inline int flat_first_cta(const Flat &f, int bh) { return (bh * f.nt) / f.T; }
__host__ __device__ inline int flat_last_cta(const Flat &f, int bh) { return ((bh + 1) * f.nt - 1) / f.T; }
__host__ __device__ inline int flat_slots(const Flat &f, int BH) { return f.n_cta + BH; }

// |k|^2 of row `row` of a ROWS-row, 128-byte-swizzled bf16 key tile (KB column blocks of 64),
// summed in a fixed order (the same in both kernels).
template <int KB, int ROWS>
__device__ __forceinline__ float key_sq_norm(const uint8_t *tile, int row) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kb = 0; kb < KB; ++kb) {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            const uint4 w = *(const uint4 *)(tile + kb * (ROWS * 128) + sw128_offset(row, ch));
            const uint32_t u[4] = {w.x, w.y, w.z, w.w};
            // acc[i] += lo_i^2, then hi_i^2, two accumulators per paired FMA-pipe instruction
#pragma unroll
            for (int i = 0; i < 4; i += 2) {
                const float lo0 = __uint_as_float(u[i] << 16), hi0 = __uint_as_float(u[i] & 0xFFFF0000u);
                const float lo1 = __uint_as_float(u[i + 1] << 16), hi1 = __uint_as_float(u[i + 1] & 0xFFFF0000u);
                ffma2(lo0, lo1, lo0, lo1, acc[i], acc[i + 1], acc[i], acc[i + 1]);
                ffma2(hi0, hi1, hi0, hi1, acc[i], acc[i + 1], acc[i], acc[i + 1]);
            }
        }
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// ============================================================================ k_key_partials
//
// Per key tile of 64 tokens, with the m features as 128-feature halves h, one per exponent
// warpgroup, each with its own TMEM buffers (the halves never wait on each other):
//   P_h^T = W_h K_tile^T (bf16 MMA; TMEM lanes are features, columns are tokens)
//   -> warpgroup h: t = P_h^T log2e + B_j with B_j = -|k_j|^2/2 log2e + A + b_t, i.e.
//      t = u_r(k_j) log2e + A + b_t; phi' = 2^(t - D_r) rounded to fp16 into TMEM
//   -> [S_h | z_h] += phi'_h [V'_t | 2^-b_t] (fp16 MMA, A from TMEM, B the converted V tile read
//      MN-major plus one column holding 2^-b_t), accumulated in TMEM over the run.
// Stabiliser D_r (integer): set on a run's first tile so that the row's largest t is in (A+b-1, A+b];
// raised whenever a later tile's largest t would exceed 15 (fp16 holds 2^t only up to t < 16),
// the row's accumulated [S | z] being scaled by 2^-delta in TMEM. Typical inputs raise it rarely.
// V'_t = V_t 2^-b_t with b_t = clamp(e_t - 7, -8, 7) and e_t the exponent of the tile's largest
// |v|: V_t is converted bf16 -> fp16 in place, and the factor 2^b_t moved into phi' keeps every
// product phi' v' equal to 2^(A - D_r) phi v. Tokens past L get phi' = 0 and a zero ones entry.
// At the end of a run warpgroup h writes its 128 feature rows of [S_h | z_h] (fp32), D_r, and the
// rows' largest magnitude and largest D_r to the run's slot.
// Warp roles (16 warps): 0-3 convert V, write the ones column and the biases B_j; 4-7 / 8-11
// exponentials of feature half 0 / 1 and the run-end write; 12 TMA; 13 MMA issue; 14 the tile's
// largest |v|; 15 idle.
// P_h^T is double-buffered where TMEM allows (d = 64): the projection of tile g+2 runs while tile g+1
// is loaded and tile g's exponentials are computed. A buffer is released as soon as its load into
// registers has completed.
// TMEM columns: P_h^T [64 (NPB h + b), +64), phi'_h [T_PHI + 32h, +32) (fp16 pairs),
// [S_h | z_h] [T_PHI + 64 + h*ON, +ON).

struct KeyStateParams2 {
    int L, m;
    Flat f;            // 64-token tiles
    float *part;       // [slots][d+1][m]: column c of [S | z] for features 0..m-1
    float *part_D;     // [slots][m]: the run's stabiliser D_r per feature
    float *part_amax;  // [slots][8]: per (half, warp) largest |entry| of the run's rows
    float *part_Dmax;  // [slots][8]: per (half, warp) largest D_r
};

constexpr int kKeyThreads = 512;
constexpr int kKeyTile = 64;            // tokens per key tile of k_key_partials
constexpr float kKeyFeatureShift = 4.f;  // A: the run's largest phi' is about 2^(A + b_t)

template <int D>
struct KeyCfg {
    static constexpr int KB = D / 64;
    static constexpr int STAGES = D == 64 ? 6 : 3;
    static constexpr int ON = D + 16;                     // N of the state MMA: values, ones, zero padding
    static constexpr uint32_t TILE = KB * kKeyTile * 128;  // K or V tile
    static constexpr uint32_t ONES = kKeyTile * 128;
    static constexpr uint32_t STAGE = 2 * TILE + ONES;     // K tile | V tile | ones block
    static constexpr int NPB = D == 64 ? 2 : 1;              // P buffers per half (TMEM allowing)
    static constexpr uint32_t T_PHI = 128 * NPB, T_S = T_PHI + 64;
};

// t = v log2e + B_j for a row of 64 logits (in place); returns the row's largest t.
__device__ __forceinline__ float key_logits(float (&v)[64], const float *bias) {
    float a = -INFINITY, b = -INFINITY;
#pragma unroll
    for (int e = 0; e < 64; e += 4) {
        const float4 b4 = *(const float4 *)(bias + e);
        v[e] = fmaf(v[e], kLog2e, b4.x);
        v[e + 1] = fmaf(v[e + 1], kLog2e, b4.y);
        v[e + 2] = fmaf(v[e + 2], kLog2e, b4.z);
        v[e + 3] = fmaf(v[e + 3], kLog2e, b4.w);
        a = fmax3(a, v[e], v[e + 1]);
        b = fmax3(b, v[e + 2], v[e + 3]);
    }
    return fmaxf(a, b);
}

// phi' = 2^(t - D) (in place), rounded to fp16 pairs. Per 32 columns the first 32 - POLY
// exponentials go to MUFU ex2, the last POLY to the FMA-pipe polynomial.
template <int POLY>
__device__ __forceinline__ void key_features(float (&v)[64], float D, uint32_t (&hv)[32]) {
#pragma unroll
    for (int e = 0; e < 64; ++e) v[e] -= D;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
#pragma unroll
        for (int e = c * 32; e < c * 32 + 32 - POLY; ++e) v[e] = ex2_approx(v[e]);
#pragma unroll
        for (int e = c * 32 + 32 - POLY; e < c * 32 + 32; e += 2) exp2_poly_pair(v[e], v[e + 1], v[e], v[e + 1]);
#pragma unroll
        for (int e = c * 32; e < c * 32 + 32; e += 2) hv[e >> 1] = pack_f16x2(v[e], v[e + 1]);
    }
}

// Stores 32 consecutive 32-bit columns of this thread's TMEM lane (warp-collective; not waited).
__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&h)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        FAVOR_U16(h, 0), FAVOR_U16(h, 16)
        : "memory");
}

// Scales columns [0, n) of this thread's TMEM lane by s (warp-collective; n a multiple of 16;
// waited). Touches no column at or past n.
__device__ __forceinline__ void tmem_scale_row(uint32_t taddr, int n, float s) {
    for (int c0 = 0; c0 < n; c0 += 16) {
        float w[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
            "%14, %15}, [%16];"
            : "=f"(w[0]), "=f"(w[1]), "=f"(w[2]), "=f"(w[3]), "=f"(w[4]), "=f"(w[5]), "=f"(w[6]), "=f"(w[7]),
              "=f"(w[8]), "=f"(w[9]), "=f"(w[10]), "=f"(w[11]), "=f"(w[12]), "=f"(w[13]), "=f"(w[14]), "=f"(w[15])
            : "r"(taddr + c0));
        asm volatile("tcgen05.wait::ld.sync.aligned;"
                     : "+f"(w[0]), "+f"(w[1]), "+f"(w[2]), "+f"(w[3]), "+f"(w[4]), "+f"(w[5]), "+f"(w[6]), "+f"(w[7]),
                       "+f"(w[8]), "+f"(w[9]), "+f"(w[10]), "+f"(w[11]), "+f"(w[12]), "+f"(w[13]), "+f"(w[14]),
                       "+f"(w[15])::"memory");
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] *= s;
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
            "%14, %15, %16};" ::"r"(taddr + c0),
            "f"(w[0]), "f"(w[1]), "f"(w[2]), "f"(w[3]), "f"(w[4]), "f"(w[5]), "f"(w[6]), "f"(w[7]), "f"(w[8]),
            "f"(w[9]), "f"(w[10]), "f"(w[11]), "f"(w[12]), "f"(w[13]), "f"(w[14]), "f"(w[15])
            : "memory");
    }
    tmem_wait_st();
}

template <int D, int POLY>
__global__ void __launch_bounds__(kKeyThreads, 1)
k_key_partials(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
               const __grid_constant__ CUtensorMap mapW, KeyStateParams2 p) {
    using C = KeyCfg<D>;
    constexpr int KB = C::KB, STAGES = C::STAGES, ON = C::ON;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int halves = p.m / 128;
    uint8_t *sW = smem;
    uint8_t *sStage = sW + (size_t)KB * p.m * 128;
    float *sBias = (float *)(sStage + (size_t)STAGES * C::STAGE);  // [STAGES][64]
    int *sShift = (int *)(sBias + STAGES * kKeyTile);               // [STAGES] (16-int slot)
    uint64_t *bars = (uint64_t *)(sShift + 16);
    uint64_t *full = bars, *empty = full + STAGES, *vmax_full = empty + STAGES, *conv_full = vmax_full + STAGES;
    // p_full / p_free: one barrier per (half, P buffer), so no waiter can fall two phases behind
    uint64_t *w_full = conv_full + STAGES, *p_full = w_full + 1, *p_free = p_full + 4;
    uint64_t *phi_full = p_free + 4, *phi_free = phi_full + 2, *acc_full = phi_free + 2, *acc_empty = acc_full + 2;
    uint64_t *drain = acc_empty + 2, *stagger = drain + 2;
    uint32_t *tmem_slot = (uint32_t *)(stagger + 1);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    pdl_launch_dependents();  // the state image kernel may stage its launch meanwhile
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nt = p.f.nt;
    const int f0 = blockIdx.x * p.f.T, f1 = min(f0 + p.f.T, p.f.total);
    const int n = max(f1 - f0, 0);

    // The ones blocks hold zeros except the per-token entry the converter writes each tile.
    for (int i = threadIdx.x; i < STAGES * (int)(C::ONES / 16); i += kKeyThreads) {
        const int s = i / (C::ONES / 16), q = i % (C::ONES / 16);
        *(uint4 *)(sStage + (size_t)s * C::STAGE + 2 * C::TILE + q * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_async_smem();
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], halves);  // one MMA commit per feature half
            mbar_init(&vmax_full[s], 1);
            mbar_init(&conv_full[s], 128);
        }
        mbar_init(w_full, 1);
        for (int i = 0; i < 4; ++i) {
            mbar_init(&p_full[i], 1);
            mbar_init(&p_free[i], 128);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&phi_full[h], 128);
            mbar_init(&phi_free[h], 1);
            mbar_init(&acc_full[h], 1);
            mbar_init(&acc_empty[h], 128);
        }
        mbar_init(&drain[0], 1);
        mbar_init(&drain[1], 1);
        mbar_init(stagger, 128);
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
        if (warp == 12 && n > 0) {
            if (elect_one()) {
                prefetch_tensormap(&mapK);
                prefetch_tensormap(&mapV);
                prefetch_tensormap(&mapW);
                mbar_arrive_expect_tx(w_full, KB * p.m * 128);
                for (int kb = 0; kb < KB; ++kb) tma_load_2d(sW + (size_t)kb * p.m * 128, &mapW, w_full, kb * 64, 0);
            }
            __syncwarp();
            int issued = 0;
            for (int g = 0; g < n; ++g) {
                const int s = g % STAGES, fl = f0 + g;
                if (!mbar_wait_lazy(&empty[s], ((g / STAGES) & 1) ^ 1, abort_flag)) break;
                if (elect_one()) {
                    mbar_arrive_expect_tx(&full[s], 2 * C::TILE);
                    uint8_t *st = sStage + (size_t)s * C::STAGE;
                    for (int kb = 0; kb < KB; ++kb) {
                        tma_load_3d(st + kb * kKeyTile * 128, &mapK, &full[s], kb * 64, (fl % nt) * kKeyTile, fl / nt);
                        tma_load_3d(st + C::TILE + kb * kKeyTile * 128, &mapV, &full[s], kb * 64, (fl % nt) * kKeyTile,
                                    fl / nt);
                    }
                }
                __syncwarp();
                ++issued;
            }
            volatile int no_abort = 0;
            for (int i = max(issued - STAGES, 0); i < issued; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1, &no_abort);
            mbar_wait(w_full, 0, &no_abort);
        } else if (warp == 14 && n > 0) {
            // Largest |v| of each V tile (bf16 magnitudes compared as integers) -> b_t.
            for (int g = 0; g < n; ++g) {
                const int s = g % STAGES;
                if (!mbar_wait_lazy(&full[s], (g / STAGES) & 1, abort_flag)) break;
                const uint8_t *vt = sStage + (size_t)s * C::STAGE + C::TILE;
                uint32_t mx = 0;
#pragma unroll 4
                for (int q = lane; q < (int)(C::TILE / 16); q += 32) {
                    const uint4 w = *(const uint4 *)(vt + q * 16);
                    mx = __vmaxu2(mx, w.x & 0x7FFF7FFFu);
                    mx = __vmaxu2(mx, w.y & 0x7FFF7FFFu);
                    mx = __vmaxu2(mx, w.z & 0x7FFF7FFFu);
                    mx = __vmaxu2(mx, w.w & 0x7FFF7FFFu);
                }
                mx = max(mx & 0xFFFFu, mx >> 16);
                for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                if (lane == 0) {
                    const int e = (int)(mx >> 7) - 127;  // exponent of the largest |v| (-127 for an all-zero tile)
                    sShift[s] = min(max(e - 7, -8), 7);
                    // V' = V 2^-b_t is an fp16 operand: from 2^23 on (and for inf / nan) it would overflow
                    if (mx >= 0x4B00u) record_status(FAVOR_ERR_UNSUPPORTED);
                    mbar_arrive(&vmax_full[s]);
                }
                __syncwarp();
            }
        } else if ((warp == 13 || warp == 15) && n > 0 && (warp == 13 || halves == 2)) {
            // MMA issue for feature half h (warp 13: h = 0, warp 15: h = 1), by the whole converged
            // warp through the predicated issue forms, so the halves never wait on each other: per
            // tile g, first the projection of tile g + NPB into the P buffer tile g has just been
            // read out of, then the state MMA of tile g once its V tile is converted and phi' is in
            // TMEM.
            const int h = warp == 13 ? 0 : 1;
            const uint32_t idesc1 = make_idesc(128, kKeyTile, kFmtBF16, 0, 0);
            const uint32_t idesc2 = make_idesc(128, ON, kFmtF16, 0, 1);
            const uint64_t dW = make_sdesc(smem_u32(sW), 16, 1024) + (uint32_t)h * (128 * 128 / 16);
            const uint64_t dS = make_sdesc(smem_u32(sStage), 16, 1024);
            const uint64_t dV = make_sdesc(smem_u32(sStage) + C::TILE, kKeyTile * 128, 1024);
            constexpr int NPB = C::NPB;
            auto project = [&](int g) {
                const uint64_t b = dS + (uint32_t)(g % STAGES) * (C::STAGE / 16);
                const uint32_t d = tmem + (uint32_t)(h * NPB + g % NPB) * 64;
                mma_ss_x4_w(d, dW, b, idesc1, 0u, 2, 2);
                if (KB == 2) mma_ss_x4_w(d, dW + (uint32_t)p.m * 8, b + kKeyTile * 128 / 16, idesc1, 1u, 2, 2);
                mma_commit_w(&p_full[h * 2 + g % NPB]);
            };
            bool ok = mbar_wait_all(w_full, 0, abort_flag);
            for (int g = 0; ok && g < min(NPB, n); ++g) {
                ok = mbar_wait_all(&full[g % STAGES], (g / STAGES) & 1, abort_flag);
                tc_fence_after();
                if (ok) project(g);
            }
            int runs = 0;
            int pos = f0 % nt;  // tile g's index within its head
            for (int g = 0; ok && g < n; ++g) {
                const int s = g % STAGES;
                const bool first = g == 0 || pos == 0, last = g == n - 1 || pos == nt - 1;
                pos = pos + 1 == nt ? 0 : pos + 1;
                if (g + NPB < n) {
                    const int g2 = g + NPB;
                    ok = mbar_wait_all(&full[g2 % STAGES], (g2 / STAGES) & 1, abort_flag) &&
                         mbar_wait_all(&p_free[h * 2 + g % NPB], (g / NPB) & 1, abort_flag);
                    tc_fence_after();
                    if (!ok) break;
                    project(g2);
                }
                ok = mbar_wait_all(&conv_full[s], (g / STAGES) & 1, abort_flag);
                if (ok && first && runs > 0) ok = mbar_wait_all(&acc_empty[h], (runs - 1) & 1, abort_flag);
                if (ok) ok = mbar_wait_all(&phi_full[h], g & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                mma_ts_x4_w(tmem + C::T_S + h * ON, tmem + C::T_PHI + h * 32, dV + (uint32_t)s * (C::STAGE / 16), idesc2,
                            first ? 0u : 1u, 2048 / 16);
                mma_commit_w(&phi_free[h]);
                if (last) {
                    mma_commit_w(&acc_full[h]);
                    ++runs;
                }
                mma_commit_w(&empty[s]);
            }
            mma_commit_w(&drain[h]);
            volatile int no_abort = 0;
            mbar_wait_all(&drain[h], 0, &no_abort);
        }
    } else if (warp >= 4) {
        regs_inc<184>();
        const int h = (warp - 4) >> 2, row = (warp & 3) * 32 + lane;
        if (h < halves) {
            constexpr int NPB = C::NPB;
            const uint32_t lane_off = ((uint32_t)(warp & 3) * 32u) << 16;
            const uint32_t tP = tmem + lane_off + h * NPB * 64, tS = tmem + lane_off + C::T_S + h * ON;
            int runs = 0;
            float Dr = 0.f;    // this feature's stabiliser D_r in the current run
            int pos = f0 % nt;  // tile g's index within its head
            float v[64];
            if (n > 0 && mbar_wait_all(&p_full[h * 2], 0, abort_flag)) {
                tc_fence_after();
                tmem_ld64_nowait(tP, v);
            }
            // The second half starts once the first has reached its first exponentials, so the two
            // warps sharing an SM sub-partition (one per half) alternate on the MUFU pipe.
            bool go = true;
            if (h == 1 && n > 0) go = mbar_wait_all(stagger, 0, abort_flag);
            for (int g = 0; go && g < n; ++g) {
                const int s = g % STAGES, b = g % NPB;
                const bool first = g == 0 || pos == 0, last = g == n - 1 || pos == nt - 1;
                pos = pos + 1 == nt ? 0 : pos + 1;
                asm volatile("tcgen05.wait::ld.sync.aligned;" : FAVOR_RW32((&v[0])), FAVOR_RW32((&v[32]))::"memory");
                // the logits are in registers: the buffer is free for the projection of tile g + NPB
                tc_fence_before();
                mbar_arrive(&p_free[h * 2 + b]);
                if (!mbar_wait_all(&conv_full[s], (g / STAGES) & 1, abort_flag)) break;
                const float Dbase = first ? 0.f : Dr;
                const float tmax = key_logits(v, sBias + s * kKeyTile) - Dbase;
                const float lim = kKeyFeatureShift + (float)sShift[s];  // target for the row's largest t
                // new stabiliser: on a run's first tile always, later only when 2^t would overflow fp16
                const float delta = (first || tmax > 15.f) ? ceilf(tmax - lim) : 0.f;
                Dr = Dbase + delta;
                if (h == 0 && g == 0 && halves == 2) mbar_arrive(stagger);
                uint32_t hv[32];
                key_features<POLY>(v, Dr, hv);
                // prefetch the next tile's logits (its projection ran meanwhile)
                if (g + 1 < n) {
                    if (!mbar_wait_all(&p_full[h * 2 + (g + 1) % NPB], ((g + 1) / NPB) & 1, abort_flag)) break;
                    tc_fence_after();
                    tmem_ld64_nowait(tP + ((g + 1) % NPB) * 64, v);
                }
                if (g > 0 && !mbar_wait_all(&phi_free[h], (g - 1) & 1, abort_flag)) break;
                tc_fence_after();
                // a raised stabiliser rescales the row's accumulated [S | z] (the previous tile's
                // state MMA has completed: phi_free)
                if (!first && __any_sync(0xffffffffu, delta > 0.f))
                    tmem_scale_row(tS, ON, __uint_as_float((uint32_t)(127 - (int)delta) << 23));
                tmem_st32u(tmem + lane_off + C::T_PHI + h * 32, hv);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&phi_full[h]);
                if (last) {
                    if (!mbar_wait_all(&acc_full[h], runs & 1, abort_flag)) break;
                    tc_fence_after();
                    const int bh = (f0 + g) / nt;
                    const size_t rs = (size_t)blockIdx.x + bh;
                    float *dst = p.part + rs * (D + 1) * p.m + h * 128 + row;
                    float amax = 0.f;
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 64) {
                        float w[64];
                        tmem_ld64_nowait(tS + c0, w);
                        asm volatile("tcgen05.wait::ld.sync.aligned;" : FAVOR_RW32((&w[0])), FAVOR_RW32((&w[32])),
                                     FAVOR_RW32((&v[0])), FAVOR_RW32((&v[32]))::"memory");
#pragma unroll
                        for (int c = 0; c < 64; ++c) {
                            dst[(size_t)(c0 + c) * p.m] = w[c];
                            amax = fmaxf(amax, fabsf(w[c]));
                        }
                    }
                    float z;
                    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=f"(z) : "r"(tS + D));
                    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+f"(z), FAVOR_RW32((&v[0])), FAVOR_RW32((&v[32]))::"memory");
                    dst[(size_t)D * p.m] = z;
                    amax = fmaxf(amax, z);
                    p.part_D[rs * p.m + h * 128 + row] = Dr;
                    tc_fence_before();
                    mbar_arrive(&acc_empty[h]);
                    float dmax = Dr;
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
        regs_dec<80>();
        // Converter warpgroup: thread j < 64 handles token j of each tile (its |k_j|^2, bias and
        // ones entry); all 128 threads convert 4 * KB of the tile's 16-byte V chunks each.
        const int j = threadIdx.x;
        for (int g = 0; g < n; ++g) {
            const int s = g % STAGES, fl = f0 + g, t = fl % nt;
            if (!mbar_wait_lazy(&vmax_full[s], (g / STAGES) & 1, abort_flag)) break;
            uint8_t *st = sStage + (size_t)s * C::STAGE;
            const int b = sShift[s];
            const float scale = __uint_as_float((uint32_t)(127 - b) << 23);  // 2^-b
#pragma unroll
            for (int i = 0; i < 4 * KB; ++i) {
                uint4 *q = (uint4 *)(st + C::TILE + (size_t)(j + 128 * i) * 16);
                uint4 w = *q;
                uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    u[k] = pack_f16x2(__uint_as_float(u[k] << 16) * scale, __uint_as_float(u[k] & 0xFFFF0000u) * scale);
                *q = make_uint4(u[0], u[1], u[2], u[3]);
            }
            if (j < kKeyTile) {
                const bool valid = t * kKeyTile + j < p.L;
                const uint32_t ones = pack_f16x2(valid ? scale : 0.f, 0.f) & 0xFFFFu;
                *(uint16_t *)(st + 2 * C::TILE + j * 128 + ((j & 7) << 4)) = (uint16_t)ones;
                const float k2 = key_sq_norm<KB, kKeyTile>(st, j);
                sBias[s * kKeyTile + j] = valid ? fmaf(-0.5f * k2, kLog2e, kKeyFeatureShift + (float)b) : -INFINITY;
            }
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

template <int D>
static size_t key_partials_smem(int m) {
    using C = KeyCfg<D>;
    return 1024 + (size_t)C::KB * m * 128 + (size_t)C::STAGES * C::STAGE + C::STAGES * kKeyTile * 4 + 64 + 640;
}

// The register split of k_key_partials (80 + 2 x 184 + 56 per warpgroup lane) fits the 128 per
// thread it is launched with; the launch is refused unless the kernel carries exactly 128.
template <int D, int POLY>
static cudaError_t launch_key_partials_t(const CUtensorMap &mK, const CUtensorMap &mV, const CUtensorMap &mW,
                                         const KeyStateParams2 &p, cudaStream_t st) {
    static int checked = 0;
    if (checked == 0) {
        cudaFuncAttributes a{};
        checked = (cudaFuncGetAttributes(&a, k_key_partials<D, POLY>) == cudaSuccess && a.numRegs == 128) ? 1 : -1;
    }
    if (checked < 0) return cudaErrorInvalidConfiguration;
    const size_t sm = key_partials_smem<D>(p.m);
    cudaFuncSetAttribute(k_key_partials<D, POLY>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_key_partials<D, POLY><<<p.f.n_cta, kKeyThreads, sm, st>>>(mK, mV, mW, p);
    return cudaGetLastError();
}

// d = 128 (d = 64 runs on k_key_partials_wide, 128-token tiles).
cudaError_t launch_key_partials(const CUtensorMap &mK, const CUtensorMap &mV, const CUtensorMap &mW,
                                const KeyStateParams2 &p, int d, int poly_pct, cudaStream_t st) {
    if (d != 128) return cudaErrorInvalidValue;
    const int poly = poly_pct < 13 ? 0 : poly_pct < 31 ? 8 : poly_pct < 44 ? 12 : 16;
    switch (poly) {
        case 0: return launch_key_partials_t<128, 0>(mK, mV, mW, p, st);
        case 8: return launch_key_partials_t<128, 8>(mK, mV, mW, p, st);
        case 12: return launch_key_partials_t<128, 12>(mK, mV, mW, p, st);
        default: return launch_key_partials_t<128, 16>(mK, mV, mW, p, st);
    }
}

}  // namespace favor
