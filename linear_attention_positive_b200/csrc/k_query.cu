// Bidirectional state finalisation and query-side output of the bf16 tensor-core path.
//
//   k_state_finalize : sums the per-split partial states in split order into the per-head
//                      state [S | z] = (K')^T [V | 1_L] and writes it in the layout the output MMA
//                      reads (tf32, K-major, 128-byte swizzled), plus z and the key stabiliser C.
//   k_query_out      : out = D^-1 (Q' S), D = diag(Q' z) ("Fast Attention Via Positive Orthogonal
//                      Random Features", codewithpapers.app/method/favor, the FA-part and its
//                      normaliser), with Q' = exp(Q W^T - rowmax) formed in TMEM.
//
// Per-head state block (floats): [ image (m*d) | z (m) | C, 0, 0, 0 ]. The image holds S[r, c]
// (in the tf32_store form) at  (c/64)*(m*64*4) + (r/32)*(64*128) + swizzle128(row c%64, chunk (r%32)/4) + (r%4)*4  bytes:
// for each half of the value columns, m/32 blocks of 64 rows x 128 bytes.

#include "common.cuh"

namespace favor {

__host__ __device__ inline size_t state_floats(int m, int d) { return (size_t)m * d + m + 4; }

__device__ __forceinline__ uint32_t state_image_offset(int r, int c, int m) {
    const int nh = c >> 6, cc = c & 63, kb = r >> 5, ch = (r & 31) >> 2, pos = r & 3;
    return (uint32_t)nh * (m * 64 * 4) + (uint32_t)kb * (64 * 128) + sw128_offset(cc, ch) + pos * 4;
}

struct FinalizeParams {
    int m, d, n_split;
    const float *part_S;     // [BH, n_split, m, d]
    const float *part_z;     // [BH, n_split, m]
    const float *head_max;   // [BH]
    float *state;            // [BH, state_floats]
};

__global__ void __launch_bounds__(256) k_state_finalize(FinalizeParams p) {
    const int bh = blockIdx.x;
    float *st = p.state + (size_t)bh * state_floats(p.m, p.d);
    uint8_t *img = (uint8_t *)st;
    const size_t md = (size_t)p.m * p.d;
    for (size_t i = threadIdx.x; i < md; i += blockDim.x) {
        const int r = (int)(i / p.d), c = (int)(i % p.d);
        float s = 0.f;
        for (int k = 0; k < p.n_split; ++k) s += p.part_S[((size_t)bh * p.n_split + k) * md + i];
        *(float *)(img + state_image_offset(r, c, p.m)) = tf32_store(s);
    }
    for (int r = threadIdx.x; r < p.m; r += blockDim.x) {
        float z = 0.f;
        for (int k = 0; k < p.n_split; ++k) z += p.part_z[((size_t)bh * p.n_split + k) * p.m + r];
        st[md + r] = z;
    }
    if (threadIdx.x == 0) {
        st[md + p.m] = p.head_max[bh];
        st[md + p.m + 1] = 0.f;
        st[md + p.m + 2] = 0.f;
        st[md + p.m + 3] = 0.f;
    }
}

// ============================================================================ k_query_out

struct QueryParams {
    int L, d, m, tiles_per_cta;
    const float *state;  // [BH, state_floats]
    float *out;          // fp32 [BH, L, d]
};

template <int D>
struct QuerySmem {
    static constexpr int KB = D / 64, NH = D / 64;
    static constexpr uint32_t Q_TILE = KB * kTile * 128;
    static constexpr int STAGES = D == 64 ? 3 : 2;
};

template <int D>
__global__ void __launch_bounds__(512, 1)
k_query_out(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapW, QueryParams p) {
    using SM = QuerySmem<D>;
    constexpr int KB = SM::KB, NH = SM::NH, STAGES = SM::STAGES;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t img_half_bytes = (uint32_t)p.m * 64 * 4;
    uint8_t *sW = smem;                                          // KB x m x 128
    uint8_t *sImg = sW + (size_t)KB * p.m * 128;                 // m x 64 x 4 (one value half)
    float *sZ = (float *)(sImg + img_half_bytes);                // m (<= 256) in a 1024-byte slot
    uint8_t *sQ = (uint8_t *)sZ + 1024;                          // STAGES x Q_TILE
    float *sRmax = (float *)(sQ + (size_t)STAGES * SM::Q_TILE);  // 2 x 128
    float *sDen = sRmax + 256;                                   // 2 (buffer) x 2 (half) x 128
    uint64_t *bars = (uint64_t *)(sDen + 512);
    uint64_t *full = bars, *empty = bars + STAGES;
    uint64_t *w_full = empty + STAGES, *img_full = w_full + 1, *img_empty = img_full + 1;
    uint64_t *p_full = img_empty + 1, *p_free = p_full + 1;
    uint64_t *chunk_full = p_free + 1;                           // 8
    uint64_t *o_full = chunk_full + 8, *o_empty = o_full + 2;
    uint64_t *den_full = o_empty + 2, *den_empty = den_full + 2, *drain = den_empty + 2;
    uint64_t *rmax_bar = drain + 1;
    uint32_t *tmem_slot = (uint32_t *)(rmax_bar + 1);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int n_tiles_total = (p.L + kTile - 1) / kTile;
    const int t0 = blockIdx.x * p.tiles_per_cta;
    const int n_tiles = max(min(t0 + p.tiles_per_cta, n_tiles_total) - t0, 0);
    const int n_iter = NH * n_tiles;
    const int halves = p.m / 128;
    const int n_chunks = p.m / 32;
    const float *st = p.state + (size_t)bh * state_floats(p.m, D);
    const uint32_t tP = 0, tO = 256;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(w_full, 1);
        mbar_init(img_full, 1);
        mbar_init(img_empty, 1);
        mbar_init(p_full, 1);
        mbar_init(p_free, 1);
        for (int c = 0; c < 8; ++c) mbar_init(&chunk_full[c], 4);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&o_full[b], 1);
            mbar_init(&o_empty[b], 4);
            mbar_init(&den_full[b], 4 * halves);
            mbar_init(&den_empty[b], 4);
        }
        mbar_init(drain, 1);
        mbar_init(rmax_bar, 8);
        *abort_flag = 0;
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

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tensormap(&mapQ);
            prefetch_tensormap(&mapW);
            mbar_arrive_expect_tx(w_full, KB * p.m * 128 + p.m * 4);
            for (int kb = 0; kb < KB; ++kb) tma_load_2d(sW + (size_t)kb * p.m * 128, &mapW, w_full, kb * 64, 0);
            bulk_load(sZ, st + (size_t)p.m * D, p.m * 4, w_full);
            int issued = 0;
            bool ok = true;
            for (int nh = 0; ok && nh < NH; ++nh) {
                if (!mbar_wait(img_empty, (nh & 1) ^ 1, abort_flag)) break;
                mbar_arrive_expect_tx(img_full, img_half_bytes);
                const uint8_t *src = (const uint8_t *)st + (size_t)nh * img_half_bytes;
                for (uint32_t off = 0; off < img_half_bytes; off += 32768)
                    bulk_load(sImg + off, src + off, min(32768u, img_half_bytes - off), img_full);
                for (int it = 0; it < n_tiles; ++it) {
                    const int g = nh * n_tiles + it, s = g % STAGES;
                    if (!mbar_wait(&empty[s], ((g / STAGES) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], SM::Q_TILE);
                    for (int kb = 0; kb < KB; ++kb)
                        tma_load_3d(sQ + (size_t)s * SM::Q_TILE + kb * kTile * 128, &mapQ, &full[s], kb * 64,
                                    (t0 + it) * kTile, bh);
                    ++issued;
                }
            }
            for (int g = max(issued - STAGES, 0); g < issued; ++g) {
                volatile int no_abort = 0;
                mbar_wait(&full[g % STAGES], (g / STAGES) & 1, &no_abort);
            }
            volatile int no_abort_w = 0;
            mbar_wait(w_full, 0, &no_abort_w);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc1 = make_idesc(kTile, p.m, kFmtBF16, 0, 0);
            const uint32_t idesc2 = make_idesc(kTile, 64, kFmtTF32, 0, 0);
            bool ok = mbar_wait(w_full, 0, abort_flag);
            for (int nh = 0; ok && nh < NH; ++nh) {
                if (!mbar_wait(img_full, nh & 1, abort_flag)) break;
                for (int it = 0; it < n_tiles; ++it) {
                    const int g = nh * n_tiles + it, s = g % STAGES, ob = g & 1;
                    if (!mbar_wait(&full[s], (g / STAGES) & 1, abort_flag) ||
                        !mbar_wait(p_free, (g & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sQ + (size_t)s * SM::Q_TILE), b0 = smem_u32(sW);
                    for (int k = 0; k < D / 16; ++k) {
                        const int kb = k >> 2, kk = k & 3;
                        mma_f16_ss(tmem + tP, make_sdesc(a0 + kb * kTile * 128 + kk * 32, 16, 1024),
                                   make_sdesc(b0 + kb * p.m * 128 + kk * 32, 16, 1024), idesc1, k > 0);
                    }
                    mma_commit(p_full);
                    mma_commit(&empty[s]);
                    if (!mbar_wait(&o_empty[ob], ((g >> 1) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    for (int ci = 0; ci < n_chunks; ++ci) {
                        // Alternate halves so both exponent warpgroups' chunks are consumed early.
                        const int c = halves == 2 ? ((ci & 1) * 4 + (ci >> 1)) : ci;
                        if (!mbar_wait(&chunk_full[c], g & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t ib = smem_u32(sImg) + c * 64 * 128;
                        for (int kk = 0; kk < 4; ++kk)
                            mma_tf32_ts(tmem + tO + ob * 64, tmem + tP + c * 32 + kk * 8,
                                        make_sdesc(ib + kk * 32, 16, 1024), idesc2, (ci > 0 || kk > 0) ? 1u : 0u);
                    }
                    if (!ok) break;
                    mma_commit(&o_full[ob]);
                    mma_commit(p_free);
                }
                mma_commit(img_empty);
            }
            mma_commit(drain);
            volatile int no_abort = 0;
            mbar_wait(drain, 0, &no_abort);
        }
    } else if (warp >= 4 && warp < 12) {
        // Exponent warpgroups: h = feature half, thread <-> token row, columns = features.
        const int h = (warp - 4) >> 2, row = (warp & 3) * 32 + lane;
        if (h < halves) {
            for (int g = 0; g < n_iter; ++g) {
                const int ob = g & 1;
                if (!mbar_wait(p_full, g & 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t base = tmem + tP + h * 128;
                float rmax = -INFINITY;
#pragma unroll 1
                for (int c0 = 0; c0 < 128; c0 += 32) {
                    float v[32];
                    tmem_ld32(tmem_lane_addr(base, warp, c0), v);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) rmax = fmax3(rmax, v[e], v[e + 1]);
                }
                if (halves == 2) {
                    // Exchange the two halves' row maxima (bounded mbarrier, not a named barrier,
                    // so an aborting warpgroup cannot strand its partner).
                    sRmax[h * 128 + row] = rmax;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(rmax_bar);
                    if (!mbar_wait(rmax_bar, g & 1, abort_flag)) break;
                    rmax = fmaxf(sRmax[row], sRmax[128 + row]);
                }
                const float cl = rmax * kLog2e;
                float den = 0.f;
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    const uint32_t ta = tmem_lane_addr(base, warp, cc * 32);
                    float v[32];
                    tmem_ld32(ta, v);
                    const float *z = sZ + h * 128 + cc * 32;
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float ph = ex2_approx(fmaf(v[e], kLog2e, -cl));
                        den = fmaf(tf32_trunc(ph), z[e], den);
                        v[e] = ph;
                    }
                    tmem_st32(ta, v);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&chunk_full[h * 4 + cc]);
                }
                if (!mbar_wait(&den_empty[ob], ((g >> 1) & 1) ^ 1, abort_flag)) break;
                sDen[(ob * 2 + h) * 128 + row] = den;
                __syncwarp();
                if (lane == 0) mbar_arrive(&den_full[ob]);
            }
        }
    } else if (warp >= 12) {
        // Output warpgroup: out = num / den, fp32 rows to global memory.
        const int row = (warp & 3) * 32 + lane;
        for (int g = 0; g < n_iter; ++g) {
            const int ob = g & 1, nh = g / max(n_tiles, 1), it = g - nh * n_tiles;
            if (!mbar_wait(&o_full[ob], (g >> 1) & 1, abort_flag)) break;
            if (!mbar_wait(&den_full[ob], (g >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            float num[64];
            tmem_ld32(tmem_lane_addr(tmem + tO + ob * 64, warp, 0), *(float(*)[32]) & num[0]);
            tmem_ld32(tmem_lane_addr(tmem + tO + ob * 64, warp, 32), *(float(*)[32]) & num[32]);
            float den = sDen[(ob * 2) * 128 + row];
            if (halves == 2) den += sDen[(ob * 2 + 1) * 128 + row];
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&o_empty[ob]);
                mbar_arrive(&den_empty[ob]);
            }
            const int j = (t0 + it) * kTile + row;
            if (j < p.L) {
                const float inv = 1.0f / den;
                float *dst = p.out + ((size_t)bh * p.L + j) * D + nh * 64;
#pragma unroll
                for (int e = 0; e < 64; e += 4)
                    *(float4 *)(dst + e) = make_float4(num[e] * inv, num[e + 1] * inv, num[e + 2] * inv, num[e + 3] * inv);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ============================================================================ host launchers

template <int D>
static size_t query_smem(int m) {
    using SM = QuerySmem<D>;
    return 1024 + (size_t)SM::KB * m * 128 + (size_t)m * 64 * 4 + 1024 + (size_t)SM::STAGES * SM::Q_TILE +
           (256 + 512) * 4 + 512;
}

cudaError_t launch_state_finalize(const FinalizeParams &p, int BH, cudaStream_t st) {
    k_state_finalize<<<BH, 256, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_query_out(const CUtensorMap &mQ, const CUtensorMap &mW, const QueryParams &p, int BH,
                             cudaStream_t st) {
    const int n_tiles = (p.L + kTile - 1) / kTile;
    const dim3 grid((n_tiles + p.tiles_per_cta - 1) / p.tiles_per_cta, BH);
    if (p.d == 64) {
        const size_t sm = query_smem<64>(p.m);
        cudaFuncSetAttribute(k_query_out<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        k_query_out<64><<<grid, 512, sm, st>>>(mQ, mW, p);
    } else {
        const size_t sm = query_smem<128>(p.m);
        cudaFuncSetAttribute(k_query_out<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        k_query_out<128><<<grid, 512, sm, st>>>(mQ, mW, p);
    }
    return cudaGetLastError();
}

}  // namespace favor
