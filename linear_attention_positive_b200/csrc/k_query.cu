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

// One thread per state element, summing the splits in order (grid: element blocks x heads).
__global__ void __launch_bounds__(256) k_state_finalize(FinalizeParams p) {
    const int bh = blockIdx.y;
    float *st = p.state + (size_t)bh * state_floats(p.m, p.d);
    const size_t md = (size_t)p.m * p.d;
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < md) {
        const int r = (int)(i / p.d), c = (int)(i % p.d);
        const float *src = p.part_S + (size_t)bh * p.n_split * md + i;
        float s = 0.f;
        for (int k = 0; k < p.n_split; ++k) s += src[(size_t)k * md];
        *(float *)((uint8_t *)st + state_image_offset(r, c, p.m)) = tf32_store(s);
    } else if (i < md + p.m) {
        const int r = (int)(i - md);
        const float *src = p.part_z + (size_t)bh * p.n_split * p.m + r;
        float z = 0.f;
        for (int k = 0; k < p.n_split; ++k) z += src[(size_t)k * p.m];
        st[md + r] = z;
    } else if (i == md + p.m) {
        st[md + p.m] = p.head_max[bh];
        st[md + p.m + 1] = 0.f;
        st[md + p.m + 2] = 0.f;
        st[md + p.m + 3] = 0.f;
    }
}

// ============================================================================ k_query_out
//
// Persistent CTAs over a flat, head-major range of (head, 128-token tile) items. Per item the 256
// features are handled as two 128-feature halves; warpgroup h owns half h end to end:
//   P[h] = Q W_h^T (bf16 MMA, N = 128) -> row max c_h over the half -> phi_h = 2^(P log2e - c_h)
//   in place (tf32 operand) and den_h = phi_h . z_h on CUDA cores -> O_h = phi_h S_h (tf32 MMA).
// The output warpgroup combines the halves exactly: with c = max(c_0, c_1) and a_h = 2^(c_h - c),
//   out = (a_0 O_0 + a_1 O_1) / (a_0 den_0 + a_1 den_1),
// i.e. the stabiliser is the exact per-row maximum. The half buffers let the projection of one
// half overlap the exponentials of the other.
// TMEM: P[0] [0,128), P[1] [128,256), O[tile parity][half] at 256 + (2 parity + half) * 64.

struct QueryParams {
    int L, d, m, BH, tiles_per_cta;
    const float *state;  // [BH, state_floats]
    float *out;          // fp32 [BH, L, d]
};

template <int D>
struct QuerySmem {
    static constexpr int KB = D / 64, NH = D / 64;
    static constexpr uint32_t Q_TILE = KB * kTile * 128;
    static constexpr int STAGES = D == 64 ? 3 : 2;
};

// Loads 64 consecutive fp32 TMEM columns of this thread's lane and waits.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&a)[32], float (&b)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : FAVOR_REG32(a)
        : "r"(taddr));
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : FAVOR_REG32(b)
        : "r"(taddr + 32));
    asm volatile("tcgen05.wait::ld.sync.aligned;" : FAVOR_RW32(a), FAVOR_RW32(b)::"memory");
}

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
    float *sDen = (float *)(sQ + (size_t)STAGES * SM::Q_TILE);  // [2 parity][2 half][128]
    float *sCl = sDen + 512;                                     // [2 parity][2 half][128]
    uint64_t *bars = (uint64_t *)(sCl + 512);
    uint64_t *full = bars, *empty = bars + STAGES;
    uint64_t *w_full = empty + STAGES, *img_full = w_full + 1, *img_empty = img_full + 1;
    uint64_t *p_full = img_empty + 1, *p_free = p_full + 2;      // per half buffer
    uint64_t *chunk_full = p_free + 2;                           // [2 half][4 chunk]
    uint64_t *o_full = chunk_full + 8, *o_empty = o_full + 2;
    uint64_t *den_full = o_empty + 2, *den_empty = den_full + 2, *drain = den_empty + 2;
    uint32_t *tmem_slot = (uint32_t *)(drain + 1);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nt = (p.L + kTile - 1) / kTile;
    const int total = p.BH * nt;
    const int f0 = blockIdx.x * p.tiles_per_cta;
    const int f1 = min(f0 + p.tiles_per_cta, total);
    const int n_items = NH * max(f1 - f0, 0);
    const int halves = p.m / 128;
    const uint32_t tO = 256;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(w_full, 1);
        mbar_init(img_full, 1);
        mbar_init(img_empty, 1);
        for (int h = 0; h < 2; ++h) {
            mbar_init(&p_full[h], 1);
            mbar_init(&p_free[h], 1);
        }
        for (int c = 0; c < 8; ++c) mbar_init(&chunk_full[c], 4);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&o_full[b], 1);
            mbar_init(&o_empty[b], 4);
            mbar_init(&den_full[b], 4 * halves);
            mbar_init(&den_empty[b], 4);
        }
        mbar_init(drain, 1);
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

    // Item order: head runs inside [f0, f1), then value halves nh, then tiles.
    const int bh_first = f0 / nt, bh_last = (f1 - 1) / nt;

    if (warp == 0) {
        if (lane == 0 && n_items > 0) {
            prefetch_tensormap(&mapQ);
            prefetch_tensormap(&mapW);
            mbar_arrive_expect_tx(w_full, KB * p.m * 128);
            for (int kb = 0; kb < KB; ++kb) tma_load_2d(sW + (size_t)kb * p.m * 128, &mapW, w_full, kb * 64, 0);
            int g = 0, grp = 0, issued = 0;
            bool ok = true;
            for (int bh = bh_first; ok && bh <= bh_last; ++bh) {
                const int lo = max(f0, bh * nt) - bh * nt, hi = min(f1, (bh + 1) * nt) - bh * nt;
                const float *st = p.state + (size_t)bh * state_floats(p.m, D);
                for (int nh = 0; ok && nh < NH; ++nh, ++grp) {
                    if (!mbar_wait(img_empty, (grp & 1) ^ 1, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(img_full, img_half_bytes + p.m * 4);
                    const uint8_t *src = (const uint8_t *)st + (size_t)nh * img_half_bytes;
                    for (uint32_t off = 0; off < img_half_bytes; off += 32768)
                        bulk_load(sImg + off, src + off, min(32768u, img_half_bytes - off), img_full);
                    bulk_load(sZ, st + (size_t)p.m * D, p.m * 4, img_full);
                    for (int t = lo; t < hi; ++t, ++g) {
                        const int s = g % STAGES;
                        if (!mbar_wait(&empty[s], ((g / STAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
                        mbar_arrive_expect_tx(&full[s], SM::Q_TILE);
                        for (int kb = 0; kb < KB; ++kb)
                            tma_load_3d(sQ + (size_t)s * SM::Q_TILE + kb * kTile * 128, &mapQ, &full[s], kb * 64,
                                        t * kTile, bh);
                        ++issued;
                    }
                }
            }
            volatile int no_abort = 0;
            for (int i = max(issued - STAGES, 0); i < issued; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1, &no_abort);
            mbar_wait(w_full, 0, &no_abort);
            if (grp > 0) mbar_wait(img_full, (grp - 1) & 1, &no_abort);
        }
    } else if (warp == 1) {
        if (lane == 0 && n_items > 0) {
            const uint32_t idesc1 = make_idesc(kTile, 128, kFmtBF16, 0, 0);
            const uint32_t idesc2 = make_idesc(kTile, 64, kFmtTF32, 0, 0);
            bool ok = mbar_wait(w_full, 0, abort_flag);
            int g = 0, grp = 0;
            for (int bh = bh_first; ok && bh <= bh_last; ++bh) {
                const int lo = max(f0, bh * nt) - bh * nt, hi = min(f1, (bh + 1) * nt) - bh * nt;
                for (int nh = 0; ok && nh < NH; ++nh, ++grp) {
                    if (!mbar_wait(img_full, grp & 1, abort_flag)) { ok = false; break; }
                    for (int t = lo; ok && t < hi; ++t, ++g) {
                        const int s = g % STAGES, ob = g & 1;
                        if (!mbar_wait(&full[s], (g / STAGES) & 1, abort_flag)) { ok = false; break; }
                        const uint32_t a0 = smem_u32(sQ + (size_t)s * SM::Q_TILE), b0 = smem_u32(sW);
                        for (int h = 0; h < halves; ++h) {
                            if (!mbar_wait(&p_free[h], (g & 1) ^ 1, abort_flag)) { ok = false; break; }
                            tc_fence_after();
                            for (int k = 0; k < D / 16; ++k) {
                                const int kb = k >> 2, kk = k & 3;
                                mma_f16_ss(tmem + h * 128, make_sdesc(a0 + kb * kTile * 128 + kk * 32, 16, 1024),
                                           make_sdesc(b0 + kb * p.m * 128 + h * 128 * 128 + kk * 32, 16, 1024), idesc1,
                                           k > 0);
                            }
                            mma_commit(&p_full[h]);
                        }
                        if (!ok) break;
                        mma_commit(&empty[s]);
                        if (!mbar_wait(&o_empty[ob], ((g >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                        for (int h = 0; ok && h < halves; ++h) {
                            for (int c = 0; c < 4; ++c) {
                                if (!mbar_wait(&chunk_full[h * 4 + c], g & 1, abort_flag)) { ok = false; break; }
                                tc_fence_after();
                                const uint32_t ib = smem_u32(sImg) + (h * 4 + c) * 64 * 128;
                                for (int kk = 0; kk < 4; ++kk)
                                    mma_tf32_ts(tmem + tO + (ob * 2 + h) * 64, tmem + h * 128 + c * 32 + kk * 8,
                                                make_sdesc(ib + kk * 32, 16, 1024), idesc2, (c > 0 || kk > 0) ? 1u : 0u);
                            }
                            if (ok) mma_commit(&p_free[h]);
                        }
                        if (!ok) break;
                        mma_commit(&o_full[ob]);
                    }
                    mma_commit(img_empty);
                }
            }
            mma_commit(drain);
            volatile int no_abort = 0;
            mbar_wait(drain, 0, &no_abort);
        }
    } else if (warp >= 4 && warp < 12) {
        // Exponent warpgroup h: thread <-> token row, the 128 feature columns of half h.
        const int h = (warp - 4) >> 2, row = (warp & 3) * 32 + lane;
        if (h < halves) {
            const uint32_t base = tmem + h * 128;
            for (int g = 0; g < n_items; ++g) {
                const int ob = g & 1;
                if (!mbar_wait(&p_full[h], g & 1, abort_flag)) break;
                tc_fence_after();
                float rmax = -INFINITY;
#pragma unroll 1
                for (int c0 = 0; c0 < 128; c0 += 64) {
                    float a[32], b[32];
                    tmem_ld64(tmem_lane_addr(base, warp, c0), a, b);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) rmax = fmax3(rmax, fmax3(a[e], a[e + 1], b[e]), b[e + 1]);
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
                        float used;
                        v[e] = tf32_round_store(ex2_approx(fmaf(v[e], kLog2e, -cl)), used);
                        den = fmaf(used, z[e], den);
                    }
                    tmem_st32(ta, v);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&chunk_full[h * 4 + cc]);
                }
                if (!mbar_wait(&den_empty[ob], ((g >> 1) & 1) ^ 1, abort_flag)) break;
                sDen[(ob * 2 + h) * 128 + row] = den;
                sCl[(ob * 2 + h) * 128 + row] = cl;
                __syncwarp();
                if (lane == 0) mbar_arrive(&den_full[ob]);
            }
        }
    } else if (warp >= 12) {
        // Output warpgroup: combine the halves and write fp32 rows.
        const int row = (warp & 3) * 32 + lane;
        int g = 0;
        bool ok = true;
        for (int bh = bh_first; ok && n_items > 0 && bh <= bh_last; ++bh) {
            const int lo = max(f0, bh * nt) - bh * nt, hi = min(f1, (bh + 1) * nt) - bh * nt;
            for (int nh = 0; ok && nh < NH; ++nh) {
                for (int t = lo; t < hi; ++t, ++g) {
                    const int ob = g & 1;
                    if (!mbar_wait(&o_full[ob], (g >> 1) & 1, abort_flag) ||
                        !mbar_wait(&den_full[ob], (g >> 1) & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    float a0 = 1.f, a1 = 0.f, den = sDen[(ob * 2) * 128 + row];
                    if (halves == 2) {
                        const float c0 = sCl[(ob * 2) * 128 + row], c1 = sCl[(ob * 2 + 1) * 128 + row];
                        const float c = fmaxf(c0, c1);
                        a0 = ex2_approx(c0 - c);
                        a1 = ex2_approx(c1 - c);
                        den = a0 * den + a1 * sDen[(ob * 2 + 1) * 128 + row];
                    }
                    const float inv = 1.0f / den;
                    a0 *= inv;
                    a1 *= inv;
                    const int j = t * kTile + row;
                    float *dst = p.out + ((size_t)bh * p.L + j) * D + nh * 64;
#pragma unroll 1
                    for (int c0 = 0; c0 < 64; c0 += 32) {
                        float v0[32], v1[32];
                        tmem_ld32(tmem_lane_addr(tmem + tO + (ob * 2) * 64, warp, c0), v0);
                        if (halves == 2) tmem_ld32(tmem_lane_addr(tmem + tO + (ob * 2 + 1) * 64, warp, c0), v1);
                        else {
#pragma unroll
                            for (int e = 0; e < 32; ++e) v1[e] = 0.f;
                        }
                        if (j < p.L) {
#pragma unroll
                            for (int e = 0; e < 32; e += 4)
                                *(float4 *)(dst + c0 + e) =
                                    make_float4(a0 * v0[e] + a1 * v1[e], a0 * v0[e + 1] + a1 * v1[e + 1],
                                                a0 * v0[e + 2] + a1 * v1[e + 2], a0 * v0[e + 3] + a1 * v1[e + 3]);
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&o_empty[ob]);
                        mbar_arrive(&den_empty[ob]);
                    }
                }
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
           (512 + 512) * 4 + 512;
}

int num_sms() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
    }
    return n;
}

cudaError_t launch_state_finalize(const FinalizeParams &p, int BH, cudaStream_t st) {
    const size_t n = (size_t)p.m * p.d + p.m + 1;
    k_state_finalize<<<dim3((unsigned)((n + 255) / 256), BH), 256, 0, st>>>(p);
    return cudaGetLastError();
}

// Persistent launch: at most one CTA per SM, each over a contiguous head-major range of tiles.
cudaError_t launch_query_out(const CUtensorMap &mQ, const CUtensorMap &mW, QueryParams p, cudaStream_t st) {
    const int total = p.BH * ((p.L + kTile - 1) / kTile);
    p.tiles_per_cta = (total + num_sms() - 1) / num_sms();
    const dim3 grid((total + p.tiles_per_cta - 1) / p.tiles_per_cta);
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
