// Key-side kernels of the bf16 tensor-core path.
//
//   k_key_logit_max : per split of L, the maximum key logit max_{j,r} u_r(k_j) with
//                     u_r(k) = w_r.k - |k|^2/2 (the per-(batch,head) key stabiliser is the max over
//                     splits), and the per-key term -|k_j|^2/2 for the state kernel.
//   k_key_state     : per split of L, the partial state [S | z] = sum_j phi(k_j) [v_j | 1]
//                     ((K')^T V and (K')^T 1_L of the FA-part, "Fast Attention Via Positive
//                     Orthogonal Random Features", codewithpapers.app/method/favor), with
//                     phi(k) = exp(u(k) - C) and C the per-(batch,head) key maximum, which
//                     cancels in D^-1.
//
// Both kernels are warp-specialised: warp 0 issues TMA copies, warp 1 owns TMEM and issues the
// tcgen05 MMAs, the remaining warps are epilogues that move accumulators TMEM -> registers.

#include "common.cuh"

namespace favor {

// ============================================================================ k_key_logit_max
//
// D[token, r] = K_tile . W^T (bf16 x bf16 -> fp32, M = 128 tokens, N = m, K = d) into TMEM; each
// epilogue thread owns one token row, takes the row max over r and adds -|k|^2/2.

struct KeyMaxParams {
    int L, d, m, n_split, tiles_per_split;
    float *bias;       // [BH, L]    -|k_j|^2 / 2
    float *split_max;  // [BH, n_split]
};

template <int D, int STAGES>
__global__ void __launch_bounds__(192, 1)
k_key_logit_max(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapW, KeyMaxParams p) {
    constexpr int KB = D / 64;                    // 64-element (128-byte) column blocks of d
    constexpr uint32_t TILE_BYTES = KB * kTile * 128;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sW = smem;                                         // KB x m x 128 B
    uint8_t *sK = sW + (size_t)KB * p.m * 128;                  // STAGES x TILE_BYTES
    uint64_t *bars = (uint64_t *)(sK + (size_t)STAGES * TILE_BYTES);
    uint64_t *full = bars, *empty = bars + STAGES, *w_full = bars + 2 * STAGES;
    uint64_t *acc_full = w_full + 1, *acc_empty = acc_full + 2, *drain = acc_empty + 2;
    uint32_t *tmem_slot = (uint32_t *)(drain + 1);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
    float *warp_max = (float *)(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, bh = blockIdx.y;
    const int n_tiles_total = (p.L + kTile - 1) / kTile;
    const int t0 = split * p.tiles_per_split;
    const int t1 = min(t0 + p.tiles_per_split, n_tiles_total);
    const int n_tiles = max(t1 - t0, 0);
    const uint32_t tmem_cols = p.m * 2 <= 256 ? 256u : 512u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1 + 4);
        }
        mbar_init(w_full, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&mapK);
            prefetch_tensormap(&mapW);
            mbar_arrive_expect_tx(w_full, KB * p.m * 128);
            for (int kb = 0; kb < KB; ++kb) tma_load_2d(sW + (size_t)kb * p.m * 128, &mapW, w_full, kb * 64, 0);
            int issued = 0;
            for (int it = 0; it < n_tiles; ++it) {
                const int s = it % STAGES;
                if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(&full[s], TILE_BYTES);
                for (int kb = 0; kb < KB; ++kb)
                    tma_load_3d(sK + (size_t)s * TILE_BYTES + kb * kTile * 128, &mapK, &full[s], kb * 64,
                                (t0 + it) * kTile, bh);
                ++issued;
            }
            // Drain: every issued copy must land before the CTA may exit.
            for (int it = max(issued - STAGES, 0); it < issued; ++it) {
                volatile int no_abort = 0;
                mbar_wait(&full[it % STAGES], (it / STAGES) & 1, &no_abort);
            }
            volatile int no_abort_w = 0;
            mbar_wait(w_full, 0, &no_abort_w);
        }
    } else if (warp == 1) {
        // MMA issue by the whole (converged) warp through the predicated issue forms.
        const uint32_t idesc = make_idesc(kTile, p.m, kFmtBF16, 0, 0);
        bool ok = mbar_wait_all(w_full, 0, abort_flag);
        for (int it = 0; ok && it < n_tiles; ++it) {
            const int s = it % STAGES, ab = it & 1;
            if (!mbar_wait_all(&full[s], (it / STAGES) & 1, abort_flag)) break;
            if (!mbar_wait_all(&acc_empty[ab], ((it >> 1) & 1) ^ 1, abort_flag)) break;
            tc_fence_after();
            const uint32_t a0 = smem_u32(sK + (size_t)s * TILE_BYTES), b0 = smem_u32(sW);
            for (int k = 0; k < D / 16; ++k) {
                const int kb = k >> 2, kk = k & 3;
                const uint64_t ad = make_sdesc(a0 + kb * kTile * 128 + kk * 32, 16, 1024);
                const uint64_t bd = make_sdesc(b0 + kb * p.m * 128 + kk * 32, 16, 1024);
                mma_f16_ss_w(tmem + ab * p.m, ad, bd, idesc, k > 0);
            }
            mma_commit_w(&acc_full[ab]);
            mma_commit_w(&empty[s]);
        }
        mma_commit_w(drain);
        volatile int no_abort = 0;
        mbar_wait_all(drain, 0, &no_abort);
    } else {
        // Epilogue: warps 2..5 cover TMEM lane quarters 2,3,0,1; thread <-> token row.
        const int q = warp & 3, row = q * 32 + lane;
        float umax = -INFINITY;
        for (int it = 0; it < n_tiles; ++it) {
            const int s = it % STAGES, ab = it & 1;
            if (!mbar_wait(&acc_full[ab], (it >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            // |k|^2 from this token's row of the staged tile (bf16, 128-byte swizzled).
            float nrm = 0.f;
            const uint8_t *tile = sK + (size_t)s * TILE_BYTES;
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = *(const uint4 *)(tile + kb * kTile * 128 + sw128_offset(row, c));
                    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float lo = __uint_as_float(w4[e] << 16), hi = __uint_as_float(w4[e] & 0xFFFF0000u);
                        nrm = fmaf(lo, lo, nrm);
                        nrm = fmaf(hi, hi, nrm);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            float rmax = -INFINITY;
            for (int c0 = 0; c0 < p.m; c0 += 32) {
                float v[32];
                tmem_ld32(tmem_lane_addr(tmem + ab * p.m, warp, c0), v);
#pragma unroll
                for (int e = 0; e < 32; e += 2) rmax = fmax3(rmax, v[e], v[e + 1]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
            const int j = (t0 + it) * kTile + row;
            if (j < p.L) {
                const float b = -0.5f * nrm;
                p.bias[(size_t)bh * p.L + j] = b;
                umax = fmaxf(umax, rmax + b);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) umax = fmaxf(umax, __shfl_xor_sync(0xffffffffu, umax, o));
        if (lane == 0) warp_max[warp - 2] = umax;
        named_bar_sync(1, 128);
        if (warp == 2 && lane == 0) {
            const float mx = fmaxf(fmaxf(warp_max[0], warp_max[1]), fmaxf(warp_max[2], warp_max[3]));
            p.split_max[(size_t)bh * p.n_split + split] = mx;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, tmem_cols);
}

// ============================================================================ k_key_state
//
// Per 64-token sub-tile: D2[r, j] = W . K_sub^T (bf16, M = 128 features per half, N = 64 tokens);
// the epilogue (thread <-> feature r) overwrites D2 in place with phi = 2^(D2 log2e + b_j) where
// b_j = (-|k_j|^2/2 - C) log2e, and sums phi into z_r; then S[r, :] += phi(TMEM, tf32) x V_sub
// (fp32 V^T in shared memory as the K-major B operand, tf32 MMA, M = 128 features, N = d,
// K = 8 tokens per step). tf32 keeps phi and V to 11 significant bits, which the 2e-2 * RMS
// output budget needs; bf16 features would use most of it.

struct KeyStateParams {
    int L, d, m, n_split, tiles_per_split;
    const uint16_t *V;       // bf16 [BH, L, d]
    const float *bias;       // [BH, L]
    const float *split_max;  // [BH, n_split]
    float *part_S;           // [BH, n_split, m, d]
    float *part_z;           // [BH, n_split, m]
    float *head_max;         // [BH] (written by split 0)
    float *key_ref;          // NULL, or [BH]: the same maximum in log2 units (the backward's reference)
};

template <int D>
struct KeyStateSmem {
    static constexpr int KB = D / 64;
    static constexpr uint32_t K_TILE = KB * kTile * 128;         // bf16 K tile
    static constexpr uint32_t V32_SUB = 2 * D * 128;             // fp32 V^T, 64 tokens
    static constexpr int STAGES = D == 64 ? 3 : 2;
};

template <int D>
__global__ void __launch_bounds__(384, 1)
k_key_state(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapW, KeyStateParams p) {
    using SM = KeyStateSmem<D>;
    constexpr int KB = SM::KB, STAGES = SM::STAGES;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sW = smem;                                           // KB x m x 128
    uint8_t *sK = sW + (size_t)KB * p.m * 128;                    // STAGES x K_TILE
    uint8_t *sV = sK + (size_t)STAGES * SM::K_TILE;               // 2 x V32_SUB
    float *sBB = (float *)(sV + 2 * SM::V32_SUB);                 // 2 x 64
    uint64_t *bars = (uint64_t *)(sBB + 128);
    uint64_t *full = bars, *empty = bars + STAGES;
    uint64_t *w_full = empty + STAGES;
    uint64_t *d2_full = w_full + 1, *d2_empty = d2_full + 2;
    uint64_t *phi_full = d2_empty + 2, *v_full = phi_full + 2, *v_empty = v_full + 2;
    uint64_t *state_done = v_empty + 2, *drain = state_done + 1;
    uint32_t *tmem_slot = (uint32_t *)(drain + 1);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
    float *sC = (float *)(tmem_slot + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x, bh = blockIdx.y;
    const int n_tiles_total = (p.L + kTile - 1) / kTile;
    const int t0 = split * p.tiles_per_split;
    const int t1 = min(t0 + p.tiles_per_split, n_tiles_total);
    const int n_tiles = max(t1 - t0, 0);
    const int n_sub = 2 * n_tiles;
    const int halves = p.m / 128;                 // feature halves (1 or 2)
    // TMEM: D2 buffers at [0, 2*halves*64), state S at [256, 256 + halves*D).
    const uint32_t d2_cols = halves * 64;
    const uint32_t s_col = 256;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(w_full, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&d2_full[b], 1);
            mbar_init(&d2_empty[b], 1);
            mbar_init(&phi_full[b], 4 * halves);
            mbar_init(&v_full[b], 2);
            mbar_init(&v_empty[b], 1);
        }
        mbar_init(state_done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        float c = -INFINITY;
        for (int s = 0; s < p.n_split; ++s) c = fmaxf(c, p.split_max[(size_t)bh * p.n_split + s]);
        *sC = c;
        if (split == 0) p.head_max[bh] = c;
        if (split == 0 && p.key_ref != nullptr) p.key_ref[bh] = c * kLog2e;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const float Clog2 = *sC * kLog2e;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&mapK);
            prefetch_tensormap(&mapW);
            mbar_arrive_expect_tx(w_full, KB * p.m * 128);
            for (int kb = 0; kb < KB; ++kb) tma_load_2d(sW + (size_t)kb * p.m * 128, &mapW, w_full, kb * 64, 0);
            int issued = 0;
            for (int it = 0; it < n_tiles; ++it) {
                const int s = it % STAGES;
                if (!mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(&full[s], SM::K_TILE);
                for (int kb = 0; kb < KB; ++kb)
                    tma_load_3d(sK + (size_t)s * SM::K_TILE + kb * kTile * 128, &mapK, &full[s], kb * 64,
                                (t0 + it) * kTile, bh);
                ++issued;
            }
            for (int it = max(issued - STAGES, 0); it < issued; ++it) {
                volatile int no_abort = 0;
                mbar_wait(&full[it % STAGES], (it / STAGES) & 1, &no_abort);
            }
            volatile int no_abort_w = 0;
            mbar_wait(w_full, 0, &no_abort_w);
        }
    } else if (warp == 1) {
        // MMA issue by the whole (converged) warp through the predicated issue forms.
        const uint32_t idesc_p = make_idesc(128, 64, kFmtBF16, 0, 0);
        const uint32_t idesc_s = make_idesc(128, D, kFmtTF32, 0, 0);
        bool ok = mbar_wait_all(w_full, 0, abort_flag);
        // Projection of sub-tile u into D2 buffer u&1.
        auto project = [&](int u) -> bool {
            const int it = u >> 1, s = it % STAGES, hs = u & 1, b = u & 1;
            if (hs == 0 && !mbar_wait_all(&full[s], (it / STAGES) & 1, abort_flag)) return false;
            if (!mbar_wait_all(&d2_empty[b], ((u >> 1) & 1) ^ 1, abort_flag)) return false;
            tc_fence_after();
            const uint32_t kt = smem_u32(sK + (size_t)s * SM::K_TILE) + hs * 64 * 128;
            for (int h = 0; h < halves; ++h) {
                const uint32_t wa = smem_u32(sW) + h * 128 * 128;
                for (int k = 0; k < D / 16; ++k) {
                    const int kb = k >> 2, kk = k & 3;
                    const uint64_t ad = make_sdesc(wa + kb * p.m * 128 + kk * 32, 16, 1024);
                    const uint64_t bd = make_sdesc(kt + kb * kTile * 128 + kk * 32, 16, 1024);
                    mma_f16_ss_w(tmem + b * d2_cols + h * 64, ad, bd, idesc_p, k > 0);
                }
            }
            mma_commit_w(&d2_full[b]);
            if (hs == 1) mma_commit_w(&empty[s]);
            return true;
        };
        if (ok && n_sub > 0) ok = project(0);
        for (int u = 0; ok && u < n_sub; ++u) {
            if (u + 1 < n_sub && !project(u + 1)) break;
            const int b = u & 1;
            if (!mbar_wait_all(&phi_full[b], (u >> 1) & 1, abort_flag)) break;
            if (!mbar_wait_all(&v_full[b], (u >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            const uint32_t vb = smem_u32(sV + b * SM::V32_SUB);
            for (int h = 0; h < halves; ++h) {
                for (int ks = 0; ks < 8; ++ks) {
                    // K-step of 8 tokens: block ks/4 of V^T, 32-byte offset inside its rows.
                    const uint64_t bd = make_sdesc(vb + (ks >> 2) * (D * 128) + (ks & 3) * 32, 16, 1024);
                    mma_tf32_ts_w(tmem + s_col + h * D, tmem + b * d2_cols + h * 64 + ks * 8, bd, idesc_s,
                                (u > 0 || ks > 0) ? 1u : 0u);
                }
            }
            mma_commit_w(&d2_empty[b]);
            mma_commit_w(&v_empty[b]);
        }
        mma_commit_w(state_done);
        mma_commit_w(drain);
        volatile int no_abort = 0;
        mbar_wait_all(drain, 0, &no_abort);
    } else if (warp == 2 || warp == 3) {
        // V converter: the bf16 V rows of a 64-token sub-tile become the K-major tf32 operand
        // V^T: [2 blocks of 32 tokens][D value rows][32 fp32], 128-byte swizzled. Lane <-> token,
        // so the transposing 4-byte stores of a warp fill one 128-byte row without bank conflicts.
        // Also b_j = (-|k_j|^2/2 - C) log2e for the sub-tile's tokens.
        const int tok = threadIdx.x - 64;  // 0..63
        const int kb = tok >> 5, ch = (tok & 31) >> 2, pos = tok & 3;
        for (int u = 0; u < n_sub; ++u) {
            const int b = u & 1;
            if (!mbar_wait(&v_empty[b], ((u >> 1) & 1) ^ 1, abort_flag)) break;
            const int j = (t0 + (u >> 1)) * kTile + (u & 1) * 64 + tok;
            uint8_t *dst = sV + b * SM::V32_SUB + kb * (D * 128) + pos * 4;
            const uint4 *src = (const uint4 *)(p.V + ((size_t)bh * p.L + j) * D);
#pragma unroll 4
            for (int e0 = 0; e0 < D; e0 += 8) {
                uint4 v = make_uint4(0, 0, 0, 0);
                if (j < p.L) v = __ldg(src + e0 / 8);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    *(float *)(dst + sw128_offset(e0 + 2 * e, ch)) = __uint_as_float(w4[e] << 16);
                    *(float *)(dst + sw128_offset(e0 + 2 * e + 1, ch)) = __uint_as_float(w4[e] & 0xFFFF0000u);
                }
            }
            sBB[b * 64 + tok] = j < p.L ? (p.bias[(size_t)bh * p.L + j] * kLog2e - Clog2) : -INFINITY;
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&v_full[b]);
        }
    } else {
        // Feature-map epilogue: warps 4..11; half h = (warp-4)/4, TMEM lane quarter warp&3,
        // thread <-> feature r = 128 h + 32 (warp&3) + lane.
        const int h = (warp - 4) >> 2, q = warp & 3;
        const int r = h * 128 + q * 32 + lane;
        float zsum = 0.f;
        if (h < halves) {
            for (int u = 0; u < n_sub; ++u) {
                const int b = u & 1;
                if (!mbar_wait(&d2_full[b], (u >> 1) & 1, abort_flag)) break;
                if (!mbar_wait(&v_full[b], (u >> 1) & 1, abort_flag)) break;
                tc_fence_after();
                const float *bb = sBB + b * 64;
#pragma unroll
                for (int c0 = 0; c0 < 64; c0 += 32) {
                    const uint32_t ta = tmem_lane_addr(tmem + b * d2_cols + h * 64, warp, c0);
                    float v[32];
                    tmem_ld32(ta, v);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        float used;
                        v[e] = tf32_round_store(ex2_approx(fmaf(v[e], kLog2e, bb[c0 + e])), used);
                        zsum += used;
                    }
                    tmem_st32(ta, v);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&phi_full[b]);
            }
            if (mbar_wait(state_done, 0, abort_flag)) {
                tc_fence_after();
                float *dstS = p.part_S + (((size_t)bh * p.n_split + split) * p.m + r) * D;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    float v[32];
                    tmem_ld32(tmem_lane_addr(tmem + s_col + h * D, warp, c0), v);
                    if (n_sub == 0) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *(float4 *)(dstS + c0 + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                }
                p.part_z[((size_t)bh * p.n_split + split) * p.m + r] = zsum;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ============================================================================ host launchers

// Each of these kernels allocates all 512 TMEM columns, so at most one CTA may be resident per
// SM: the dynamic shared-memory request is padded to more than half of the SM's capacity.
constexpr size_t kOneCtaPerSmSmem = 120 * 1024;

template <int D, int STAGES>
static size_t key_max_smem(int m) {
    return std::max(kOneCtaPerSmSmem, 1024 + (size_t)(D / 64) * m * 128 + (size_t)STAGES * (D / 64) * kTile * 128 + 256);
}
template <int D>
static size_t key_state_smem(int m) {
    using SM = KeyStateSmem<D>;
    return std::max(kOneCtaPerSmSmem,
                    1024 + (size_t)SM::KB * m * 128 + (size_t)SM::STAGES * SM::K_TILE + 2 * SM::V32_SUB + 512 + 256);
}

cudaError_t launch_key_logit_max(const CUtensorMap &mK, const CUtensorMap &mW, const KeyMaxParams &p, int BH,
                                  cudaStream_t st) {
    const dim3 grid(p.n_split, BH);
    if (p.d == 64) {
        const size_t sm = key_max_smem<64, 4>(p.m);
        cudaFuncSetAttribute(k_key_logit_max<64, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        k_key_logit_max<64, 4><<<grid, 192, sm, st>>>(mK, mW, p);
    } else {
        const size_t sm = key_max_smem<128, 3>(p.m);
        cudaFuncSetAttribute(k_key_logit_max<128, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        k_key_logit_max<128, 3><<<grid, 192, sm, st>>>(mK, mW, p);
    }
    return cudaGetLastError();
}

cudaError_t launch_key_state(const CUtensorMap &mK, const CUtensorMap &mW, const KeyStateParams &p, int BH,
                             cudaStream_t st) {
    const dim3 grid(p.n_split, BH);
    if (p.d == 64) {
        const size_t sm = key_state_smem<64>(p.m);
        cudaFuncSetAttribute(k_key_state<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        k_key_state<64><<<grid, 384, sm, st>>>(mK, mW, p);
    } else {
        const size_t sm = key_state_smem<128>(p.m);
        cudaFuncSetAttribute(k_key_state<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        k_key_state<128><<<grid, 384, sm, st>>>(mK, mW, p);
    }
    return cudaGetLastError();
}

}  // namespace favor
