// Causal (masked, j <= i) FAVOR+ forward on the bf16 tensor-core path.
//
// The masked FA-part ("Random Features for Efficient Attention Approximation", thesis abstract:
// masked self-attention; the FA-part of "Fast Attention Via Positive Orthogonal Random Features",
// codewithpapers.app/method/favor, with prefix sums in place of the full sums):
//   out_i = phi(q_i)^T S_i / phi(q_i)^T z_i,   S_i = sum_{j<=i} phi(k_j) v_j^T,  z_i = sum_{j<=i} phi(k_j).
//
// Sequence parallelism: the sequence of each head is cut into segments (runs of 128-token
// tiles). k_key_state (shared with the bidirectional path) gives each segment's aggregate
// [S | z]; k_state_scan turns them into exclusive prefixes; k_causal_out walks each segment's
// tiles in order from that prefix:
//   out_tile = ( phi(Q_t) S_<t + mask(phi(Q_t) phi(K_t)^T) V_t ) / ( phi(Q_t) z_<t + rowsum(mask(...)) ),
//   S_<t+1 = S_<t + phi(K_t)^T V_t.
// k_causal_prefix_* recompute the first tokens of every head in fp32 on CUDA cores: there the
// output is a weighted mean of few values, its magnitude is far above the RMS of a long output,
// and the 11-bit tf32 operands alone would use up the error budget.

#include "common.cuh"

namespace favor {

// ============================================================================ k_state_scan

struct ScanParams {
    int m, d, n_split;
    const float *part_S;    // [BH, n_split, m, d]
    const float *part_z;    // [BH, n_split, m]
    const float *head_max;  // [BH]
    float *seg_state;       // [BH, n_split, state_floats]: exclusive prefix per segment
};

// One thread per position of the state image (so the image writes are coalesced), walking the
// segments in order with the loads of four segments in flight (grid: element blocks x heads).
__global__ void __launch_bounds__(256) k_state_scan(ScanParams p) {
    const int bh = blockIdx.y;
    const size_t md = (size_t)p.m * p.d, sf = state_floats(p.m, p.d);
    float *base = p.seg_state + (size_t)bh * p.n_split * sf;
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < md) {
        // image byte offset 4i -> (r, c), the inverse of state_image_offset
        const uint32_t B = (uint32_t)i * 4u, half = (uint32_t)p.m * 256u;
        const uint32_t nh = B / half, rem = B % half, kb = rem / 8192u, rem2 = rem % 8192u;
        const uint32_t cc = rem2 / 128u, phys = (rem2 % 128u) / 16u, pos = (rem2 % 16u) / 4u;
        const int r = (int)(kb * 32u + ((phys ^ (cc & 7u)) * 4u) + pos), c = (int)(nh * 64u + cc);
        const float *src = p.part_S + (size_t)bh * p.n_split * md + (size_t)r * p.d + c;
        float run = 0.f;
        int sg = 0;
        for (; sg + 4 <= p.n_split; sg += 4) {
            const float a0 = src[(size_t)sg * md], a1 = src[(size_t)(sg + 1) * md];
            const float a2 = src[(size_t)(sg + 2) * md], a3 = src[(size_t)(sg + 3) * md];
            base[(size_t)sg * sf + i] = tf32_store(run);
            run += a0;
            base[(size_t)(sg + 1) * sf + i] = tf32_store(run);
            run += a1;
            base[(size_t)(sg + 2) * sf + i] = tf32_store(run);
            run += a2;
            base[(size_t)(sg + 3) * sf + i] = tf32_store(run);
            run += a3;
        }
        for (; sg < p.n_split; ++sg) {
            base[(size_t)sg * sf + i] = tf32_store(run);
            run += src[(size_t)sg * md];
        }
    } else if (i < md + p.m) {
        const int r = (int)(i - md);
        const float *src = p.part_z + (size_t)bh * p.n_split * p.m + r;
        float run = 0.f;
        for (int sg = 0; sg < p.n_split; ++sg) {
            base[(size_t)sg * sf + md + r] = run;
            run += src[(size_t)sg * p.m];
        }
    } else if (i < md + p.m + p.n_split) {
        float *t = base + (i - md - p.m) * sf + md + p.m;
        t[0] = p.head_max[bh];
        t[1] = t[2] = t[3] = 0.f;
    }
}

struct PrefixParams {
    int L, d, m, P;              // P = tokens per head recomputed exactly
    const uint16_t *Q, *K, *V;   // bf16 [BH, L, d]
    const uint16_t *W;           // bf16 [m, d]
    const float *bias;           // [BH, L]  -|k|^2/2
    const float *head_max;       // [BH]
    float *phiQ, *phiK;          // [BH, P, m] fp32 scratch
    float *out;                  // fp32 [BH, L, d]
};

__device__ __forceinline__ float bf16_to_f(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// phi(q) = exp(w.q - max_r w.q) and phi(k) = exp(w.k - |k|^2/2 - C) in fp32 for the first P tokens
// of each head. CTA per (32 tokens, head); thread r computes feature r (its W row in registers)
// for all 32 tokens; the per-token max over features goes through shared memory.
__global__ void __launch_bounds__(256) k_causal_prefix_features(PrefixParams p) {
    __shared__ uint16_t xq[32][64], xk[32][64];
    __shared__ float su[32][256], smax[32];
    const int bh = blockIdx.y, j0 = blockIdx.x * 32, t = threadIdx.x;
    for (int idx = t; idx < 32 * 64; idx += 256) {
        const int a = idx >> 6, e = idx & 63;
        const int j = j0 + a;
        const size_t row = ((size_t)bh * p.L + j) * p.d;
        xq[a][e] = (j < p.P && e < p.d) ? p.Q[row + e] : (uint16_t)0;
        xk[a][e] = (j < p.P && e < p.d) ? p.K[row + e] : (uint16_t)0;
    }
    __syncthreads();
    const float C = p.head_max[bh];
    if (t < p.m) {
        float w[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) w[e] = e < p.d ? bf16_to_f(p.W[(size_t)t * p.d + e]) : 0.f;
        for (int a = 0; a < 32; ++a) {
            float sq0 = 0.f, sq1 = 0.f, sk0 = 0.f, sk1 = 0.f;
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
                sq0 = fmaf(w[e], bf16_to_f(xq[a][e]), sq0);
                sq1 = fmaf(w[e + 1], bf16_to_f(xq[a][e + 1]), sq1);
                sk0 = fmaf(w[e], bf16_to_f(xk[a][e]), sk0);
                sk1 = fmaf(w[e + 1], bf16_to_f(xk[a][e + 1]), sk1);
            }
            su[a][t] = sq0 + sq1;
            const int j = j0 + a;
            if (j < p.P) p.phiK[((size_t)bh * p.P + j) * p.m + t] = expf(sk0 + sk1 + p.bias[(size_t)bh * p.L + j] - C);
        }
    }
    __syncthreads();
    {
        const int warp = t >> 5, lane = t & 31;
        for (int a = warp * 4; a < warp * 4 + 4; ++a) {
            float mx = -INFINITY;
            for (int r = lane; r < p.m; r += 32) mx = fmaxf(mx, su[a][r]);
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (lane == 0) smax[a] = mx;
        }
    }
    __syncthreads();
    if (t < p.m)
        for (int a = 0; a < 32; ++a) {
            const int j = j0 + a;
            if (j < p.P) p.phiQ[((size_t)bh * p.P + j) * p.m + t] = expf(su[a][t] - smax[a]);
        }
}

// Masked attention over the first P tokens in fp32: CTA per (64 queries, head), 256 threads.
// Per 64-key block up to the diagonal: scores S = phi(Q) phi(K)^T (4 x 4 per thread, features in
// 32-wide slices through shared memory), the mask j <= i, then num += S V and den += rowsum(S)
// (4 queries x 4 value columns per thread).
__global__ void __launch_bounds__(256) k_causal_prefix_attn(PrefixParams p) {
    // the feature slices (score phase) and the masked scores (output phase) share one buffer
    __shared__ __align__(16) float buf[64 * 65];
    __shared__ __align__(16) float sv[64][64];  // V block
    float(*aq)[64] = (float(*)[64])buf;         // [32 features][64 queries]
    float(*ak)[64] = (float(*)[64])(buf + 32 * 64);
    float(*ss)[65] = (float(*)[65])buf;         // [64 queries][64 keys + pad]
    const int bh = blockIdx.y, i0 = blockIdx.x * 64, t = threadIdx.x;
    const int ti = (t >> 4) * 4, tj = (t & 15) * 4;  // this thread's 4 x 4 score block / 4 x 4 output block
    float num[4][4], den[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        den[a] = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) num[a][c] = 0.f;
    }
    const float *phq = p.phiQ + (size_t)bh * p.P * p.m;
    const float *phk = p.phiK + (size_t)bh * p.P * p.m;
    for (int j0 = 0; j0 <= i0 && j0 < p.P; j0 += 64) {
        float sc[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) sc[a][b] = 0.f;
        for (int f0 = 0; f0 < p.m; f0 += 32) {
            __syncthreads();
            for (int idx = t; idx < 64 * 32; idx += 256) {
                const int a = idx >> 5, f = idx & 31;
                aq[f][a] = (i0 + a < p.P) ? phq[(size_t)(i0 + a) * p.m + f0 + f] : 0.f;
                ak[f][a] = (j0 + a < p.P) ? phk[(size_t)(j0 + a) * p.m + f0 + f] : 0.f;
            }
            __syncthreads();
#pragma unroll 8
            for (int f = 0; f < 32; ++f) {
                const float4 q4 = *(const float4 *)&aq[f][ti], k4 = *(const float4 *)&ak[f][tj];
                const float qv[4] = {q4.x, q4.y, q4.z, q4.w}, kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) sc[a][b] = fmaf(qv[a], kv[b], sc[a][b]);
            }
        }
        __syncthreads();
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) ss[ti + a][tj + b] = (j0 + tj + b <= i0 + ti + a) ? sc[a][b] : 0.f;
        for (int idx = t; idx < 64 * 64; idx += 256) {
            const int a = idx >> 6, e = idx & 63;
            sv[a][e] = (j0 + a < p.P && e < p.d) ? bf16_to_f(p.V[((size_t)bh * p.L + j0 + a) * p.d + e]) : 0.f;
        }
        __syncthreads();
        for (int j = 0; j < 64; ++j) {
            const float4 v4 = *(const float4 *)&sv[j][tj];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const float sa = ss[ti + a][j];
                num[a][0] = fmaf(sa, v4.x, num[a][0]);
                num[a][1] = fmaf(sa, v4.y, num[a][1]);
                num[a][2] = fmaf(sa, v4.z, num[a][2]);
                num[a][3] = fmaf(sa, v4.w, num[a][3]);
                den[a] += sa;
            }
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int i = i0 + ti + a;
        if (i < p.P && i < p.L && tj < p.d) {
            float *o = p.out + ((size_t)bh * p.L + i) * p.d + tj;
            *(float4 *)o = make_float4(num[a][0] / den[a], num[a][1] / den[a], num[a][2] / den[a], num[a][3] / den[a]);
        }
    }
}

// ============================================================================ k_causal_out
//
// One CTA per (batch-head, segment), 256 threads (two warpgroups), phases in sequence per tile.
// TMEM (512 columns):  R0 [0,128)   phi(Q) half h (fp32/tf32), later the state update dS_h
//                      R1 [128,256) phi(K)^T half h (features on lanes, tokens on columns)
//                      R2 [256,384) intra-tile scores A (q rows, k columns)
//                      R3 [384,448) output accumulator (d = 64)
// The full query projection for the per-row max uses R0..R1 before the halves.
// Shared: W (bf16), the running state S as the tf32 K-major operand image and z (fp32), the Q/K
// tiles (bf16, TMA), V^T (tf32 K-major), two 32-feature slots of phi(K) as the K-major B operand
// of the score MMA.

struct CausalParams {
    int L, d, m, tiles_per_split, P_exact;
    const uint16_t *V;        // bf16 [BH, L, d]
    const float *bias;        // [BH, L]
    const float *seg_state;   // [BH, n_split, state_floats]
    int n_split;
    float *out;               // fp32 [BH, L, d]
};

constexpr int kCausalThreads = 256;

template <int D>
struct CausalSmem {
    static constexpr uint32_t W_BYTES = (D / 64) * 256 * 128;   // m <= 256
    static constexpr uint32_t S_BYTES = 256 * D * 4;
    static constexpr uint32_t QK_BYTES = (D / 64) * kTile * 128;
    static constexpr uint32_t VT_BYTES = kTile * D * 4;
    static constexpr uint32_t KB_SLOT = kTile * 128;            // 128 tokens x 32 fp32
};

template <int D>
__global__ void __launch_bounds__(kCausalThreads, 1)
k_causal_out(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
             const __grid_constant__ CUtensorMap mapW, CausalParams p) {
    using SM = CausalSmem<D>;
    constexpr int KB = D / 64;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sW = smem;
    uint8_t *sS = sW + SM::W_BYTES;                 // state image (m x D fp32, K-major tf32)
    uint8_t *sQ = sS + SM::S_BYTES;
    uint8_t *sK = sQ + SM::QK_BYTES;
    uint8_t *sVt = sK + SM::QK_BYTES;               // [4 blocks of 32 tokens][D rows][32 fp32]
    uint8_t *sKB = sVt + SM::VT_BYTES;              // 2 slots x [128 tokens][32 fp32]
    float *sZ = (float *)(sKB + 2 * SM::KB_SLOT);   // m
    float *sRow = sZ + 256;                          // 2 x 128: per-row partials (max / sums)
    float *sC = sRow + 256;                          // 128: query row max
    float *sDen = sC + 128;                          // 128: phi(q).z_<t
    float *sBB = sDen + 128;                         // 128: (-|k|^2/2 - C) log2e
    float *sZp = sBB + 128;                          // 2 x 256: z partials of this tile
    uint64_t *bars = (uint64_t *)(sZp + 512);
    uint64_t *tma_bar = bars, *mma_bar = bars + 1;
    uint32_t *tmem_slot = (uint32_t *)(bars + 2);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = warp >> 2;                        // warpgroup: column half of every epilogue
    const int row = (warp & 3) * 32 + lane;          // TMEM lane owned by this thread
    const int split = blockIdx.x, bh = blockIdx.y;
    const int n_tiles_total = (p.L + kTile - 1) / kTile;
    const int t0 = split * p.tiles_per_split;
    const int n_tiles = max(min(t0 + p.tiles_per_split, n_tiles_total) - t0, 0);
    const int m = p.m, halves = m / 128;
    const uint32_t R0 = 0, R1 = 128, R2 = 256, R3 = 384;
    const float *seg = p.seg_state + ((size_t)bh * p.n_split + split) * state_floats(m, D);
    uint32_t tma_phase = 0, mma_phase = 0;
    bool ok = true;

    if (tid == 0) {
        mbar_init(tma_bar, 1);
        mbar_init(mma_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const float Clog2 = seg[(size_t)m * D + m] * kLog2e;

    // Segment start: W, the state prefix image and z.
    if (tid == 0) {
        prefetch_tensormap(&mapQ);
        prefetch_tensormap(&mapK);
        mbar_arrive_expect_tx(tma_bar, SM::W_BYTES / 256 * m + (uint32_t)m * D * 4 + m * 4);
        for (int kb = 0; kb < KB; ++kb) tma_load_2d(sW + (size_t)kb * m * 128, &mapW, tma_bar, kb * 64, 0);
        for (uint32_t off = 0; off < (uint32_t)m * D * 4; off += 32768)
            bulk_load(sS + off, (const uint8_t *)seg + off, min(32768u, (uint32_t)m * D * 4 - off), tma_bar);
        bulk_load(sZ, seg + (size_t)m * D, m * 4, tma_bar);
    }
    ok = mbar_wait(tma_bar, tma_phase, abort_flag);
    tma_phase ^= 1;

    auto mma_sync = [&]() -> bool {  // all threads: wait for the MMAs committed by thread 0
        const bool r = mbar_wait(mma_bar, mma_phase, abort_flag);
        mma_phase ^= 1;
        tc_fence_after();
        return r;
    };
    auto to_mma = [&]() {  // epilogue writes (TMEM and shared) before MMAs issued by thread 0
        tmem_wait_st();
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    };

    for (int it = 0; ok && it < n_tiles; ++it) {
        const int tile = t0 + it, j0 = tile * kTile;
        // ---- loads: Q, K tiles by TMA; V^T (tf32) and the key biases by the threads
        if (tid == 0) {
            mbar_arrive_expect_tx(tma_bar, 2 * SM::QK_BYTES);
            for (int kb = 0; kb < KB; ++kb) {
                tma_load_3d(sQ + kb * kTile * 128, &mapQ, tma_bar, kb * 64, j0, bh);
                tma_load_3d(sK + kb * kTile * 128, &mapK, tma_bar, kb * 64, j0, bh);
            }
        }
        {
            const int tok = tid & 127, vh = tid >> 7;  // value half
            const int j = j0 + tok;
            const int kb = tok >> 5, ch = (tok & 31) >> 2, pos = tok & 3;
            uint8_t *dst = sVt + kb * (D * 128) + pos * 4;
            const uint4 *src = (const uint4 *)(p.V + ((size_t)bh * p.L + j) * D);
            for (int e0 = vh * (D / 2); e0 < (vh + 1) * (D / 2); e0 += 8) {
                uint4 v = make_uint4(0, 0, 0, 0);
                if (j < p.L) v = __ldg(src + e0 / 8);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    *(float *)(dst + sw128_offset(e0 + 2 * e, ch)) = __uint_as_float(w4[e] << 16);
                    *(float *)(dst + sw128_offset(e0 + 2 * e + 1, ch)) = __uint_as_float(w4[e] & 0xFFFF0000u);
                }
            }
            if (vh == 0) sBB[tok] = j < p.L ? p.bias[(size_t)bh * p.L + j] * kLog2e - Clog2 : -INFINITY;
        }
        if (!(ok = mbar_wait(tma_bar, tma_phase, abort_flag))) break;
        tma_phase ^= 1;
        to_mma();

        // ---- 1. full query projection (per-row max)
        if (tid == 0) {
            const uint32_t idesc = make_idesc(kTile, m, kFmtBF16, 0, 0);
            for (int k = 0; k < D / 16; ++k)
                mma_f16_ss(tmem + R0, make_sdesc(smem_u32(sQ) + (k >> 2) * kTile * 128 + (k & 3) * 32, 16, 1024),
                           make_sdesc(smem_u32(sW) + (k >> 2) * m * 128 + (k & 3) * 32, 16, 1024), idesc, k > 0);
            mma_commit(mma_bar);
        }
        if (!(ok = mma_sync())) break;
        {
            float rmax = -INFINITY;
            for (int c0 = wg * (m / 2); c0 < (wg + 1) * (m / 2); c0 += 32) {
                float v[32];
                tmem_ld32(tmem_lane_addr(tmem + R0, warp, c0), v);
#pragma unroll
                for (int e = 0; e < 32; e += 2) rmax = fmax3(rmax, v[e], v[e + 1]);
            }
            sRow[wg * 128 + row] = rmax;
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            if (wg == 0) {
                sC[row] = fmaxf(sRow[row], sRow[128 + row]) * kLog2e;
                sDen[row] = 0.f;
            }
            __syncthreads();
        }

        for (int h = 0; h < halves; ++h) {
            // ---- 2a. projections of feature half h: phi(Q)_h (tokens x 128) and phi(K)_h^T
            if (tid == 0) {
                const uint32_t id_q = make_idesc(kTile, 128, kFmtBF16, 0, 0);
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t kq = (k >> 2) * kTile * 128 + (k & 3) * 32;
                    const uint32_t kw = (k >> 2) * m * 128 + h * 128 * 128 + (k & 3) * 32;
                    mma_f16_ss(tmem + R0, make_sdesc(smem_u32(sQ) + kq, 16, 1024),
                               make_sdesc(smem_u32(sW) + kw, 16, 1024), id_q, k > 0);
                    mma_f16_ss(tmem + R1, make_sdesc(smem_u32(sW) + kw, 16, 1024),
                               make_sdesc(smem_u32(sK) + kq, 16, 1024), id_q, k > 0);
                }
                mma_commit(mma_bar);
            }
            if (!(ok = mma_sync())) break;
            // ---- 2b. exponentials in place (tf32 operands), phi(q).z_<t, z partials, phi(K) B slots
            {
                const float cl = sC[row];
                float den = 0.f;
                for (int c0 = wg * 64; c0 < wg * 64 + 64; c0 += 32) {
                    const uint32_t ta = tmem_lane_addr(tmem + R0, warp, c0);
                    float v[32];
                    tmem_ld32(ta, v);
                    const float *z = sZ + h * 128 + c0;
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        float used;
                        v[e] = tf32_round_store(ex2_approx(fmaf(v[e], kLog2e, -cl)), used);
                        den = fmaf(used, z[e], den);
                    }
                    tmem_st32(ta, v);
                }
                atomicAdd(&sDen[row], den);
            }
            {
                // thread <-> feature f = 128 h + row; columns = tokens [64 wg, 64 wg + 64)
                float zs = 0.f;
                for (int c0 = wg * 64; c0 < wg * 64 + 64; c0 += 32) {
                    const uint32_t ta = tmem_lane_addr(tmem + R1, warp, c0);
                    float v[32];
                    tmem_ld32(ta, v);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        float used;
                        v[e] = tf32_round_store(ex2_approx(fmaf(v[e], kLog2e, sBB[c0 + e])), used);
                        zs += used;
                    }
                    tmem_st32(ta, v);
                }
                sZp[wg * 256 + h * 128 + row] = zs;
            }
            // ---- 2c. state term O (+)= phi(Q)_h S_<t[half h] (reads the state image before it changes)
            to_mma();
            if (tid == 0) {
                const uint32_t id_o = make_idesc(kTile, D, kFmtTF32, 0, 0);
                for (int k8 = 0; k8 < 16; ++k8) {
                    const int f0 = h * 128 + k8 * 8;
                    const uint32_t b = smem_u32(sS) + (f0 >> 5) * (D * 128) + (k8 & 3) * 32;
                    mma_tf32_ts(tmem + R3, tmem + R0 + k8 * 8, make_sdesc(b, 16, 1024), id_o, (h > 0 || k8 > 0) ? 1u : 0u);
                }
                mma_commit(mma_bar);
            }
            // ---- 2d. intra scores A (+)= phi(Q)_h phi(K)_h^T, 32 features per slot, two slots
            for (int cp = 0; cp < 2; ++cp) {
                if (!(ok = mma_sync())) break;  // previous MMAs done: slots and state image free
                // phi(K) chunks 2cp, 2cp+1 of half h -> slots: row = token, 32 features
                {
                    const int f = row;                       // feature within the half
                    const int chunk = f >> 5;
                    if ((chunk >> 1) == cp) {
                        uint8_t *slot = sKB + (chunk & 1) * SM::KB_SLOT;
                        const int fc = f & 31, ch = fc >> 2, pos = fc & 3;
                        for (int c0 = wg * 64; c0 < wg * 64 + 64; c0 += 32) {
                            float v[32];
                            tmem_ld32(tmem_lane_addr(tmem + R1, warp, c0), v);
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                *(float *)(slot + sw128_offset(c0 + e, ch) + pos * 4) = v[e];
                        }
                    }
                }
                to_mma();
                if (tid == 0) {
                    const uint32_t id_a = make_idesc(kTile, kTile, kFmtTF32, 0, 0);
                    for (int s = 0; s < 2; ++s) {
                        const int chunk = 2 * cp + s;
                        for (int k8 = 0; k8 < 4; ++k8)
                            mma_tf32_ts(tmem + R2, tmem + R0 + chunk * 32 + k8 * 8,
                                        make_sdesc(smem_u32(sKB) + s * SM::KB_SLOT + k8 * 32, 16, 1024), id_a,
                                        (h > 0 || chunk > 0 || k8 > 0) ? 1u : 0u);
                    }
                    mma_commit(mma_bar);
                }
            }
            if (!ok) break;
            if (!(ok = mma_sync())) break;
            // ---- 2e. state update of half h: dS_h = phi(K)_h^T V^T into R0 (phi(Q)_h consumed)
            if (tid == 0) {
                const uint32_t id_s = make_idesc(128, D, kFmtTF32, 0, 0);
                for (int k8 = 0; k8 < 16; ++k8) {
                    const uint32_t b = smem_u32(sVt) + (k8 >> 2) * (D * 128) + (k8 & 3) * 32;
                    mma_tf32_ts(tmem + R0, tmem + R1 + k8 * 8, make_sdesc(b, 16, 1024), id_s, k8 > 0);
                }
                mma_commit(mma_bar);
            }
            if (!(ok = mma_sync())) break;
            // S image[half h] += dS_h (thread <-> feature, value columns split by warpgroup)
            {
                const int f = h * 128 + row;
                const int kb = f >> 5, ch = (f & 31) >> 2, pos = f & 3;
                for (int c0 = wg * (D / 2); c0 < (wg + 1) * (D / 2); c0 += 32) {
                    float v[32];
                    tmem_ld32(tmem_lane_addr(tmem + R0, warp, c0), v);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        float *s = (float *)(sS + kb * (D * 128) + sw128_offset(c0 + e, ch) + pos * 4);
                        *s = tf32_store(tf32_load(*s) + v[e]);
                    }
                }
            }
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
        }
        if (!ok) break;
        // z += this tile's key sums (after every phi(q).z_<t of the tile used the old z)
        for (int f = tid; f < m; f += kCausalThreads) sZ[f] += sZp[f] + sZp[256 + f];
        // ---- 3. mask the scores (k > q or k past L -> 0), row sums, tf32 A operand in place
        {
            const int qi = row;
            float rs = 0.f;
            for (int c0 = wg * 64; c0 < wg * 64 + 64; c0 += 32) {
                const uint32_t ta = tmem_lane_addr(tmem + R2, warp, c0);
                float v[32];
                tmem_ld32(ta, v);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int kj = c0 + e;
                    float used;
                    v[e] = tf32_round_store((kj <= qi && j0 + kj < p.L) ? v[e] : 0.f, used);
                    rs += used;
                }
                tmem_st32(ta, v);
            }
            sRow[wg * 128 + row] = rs;
        }
        to_mma();
        // ---- 4. O += A V
        if (tid == 0) {
            const uint32_t id_o = make_idesc(kTile, D, kFmtTF32, 0, 0);
            for (int k8 = 0; k8 < 16; ++k8) {
                const uint32_t b = smem_u32(sVt) + (k8 >> 2) * (D * 128) + (k8 & 3) * 32;
                mma_tf32_ts(tmem + R3, tmem + R2 + k8 * 8, make_sdesc(b, 16, 1024), id_o, 1u);
            }
            mma_commit(mma_bar);
        }
        if (!(ok = mma_sync())) break;
        // ---- 5. out = O / (phi(q).z_<t + rowsum(A)); rows before P_exact come from the exact pass
        {
            const int i = j0 + row;
            const float den = sDen[row] + sRow[row] + sRow[128 + row];
            const float inv = 1.0f / den;
            for (int c0 = wg * (D / 2); c0 < (wg + 1) * (D / 2); c0 += 32) {
                float v[32];
                tmem_ld32(tmem_lane_addr(tmem + R3, warp, c0), v);
                if (i < p.L && i >= p.P_exact) {
                    float *o = p.out + ((size_t)bh * p.L + i) * D + c0;
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *(float4 *)(o + e) = make_float4(v[e] * inv, v[e + 1] * inv, v[e + 2] * inv, v[e + 3] * inv);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    // Drain outstanding copies and MMAs before the CTA exits and TMEM is released (bounded).
    if (tid == 0) {
        volatile int no_abort = 0;
        if (!ok) mbar_wait(tma_bar, tma_phase, &no_abort);  // a copy may still be in flight
        mma_commit(mma_bar);
        mbar_wait(mma_bar, mma_phase, &no_abort);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ============================================================================ host launchers

template <int D>
static size_t causal_smem() {
    using SM = CausalSmem<D>;
    return 1024 + SM::W_BYTES + SM::S_BYTES + 2 * SM::QK_BYTES + SM::VT_BYTES + 2 * SM::KB_SLOT +
           (256 + 256 + 128 * 3 + 512) * 4 + 256;
}

cudaError_t launch_state_scan(const ScanParams &p, int BH, cudaStream_t st) {
    const size_t n = (size_t)p.m * p.d + p.m + p.n_split;
    k_state_scan<<<dim3((unsigned)((n + 255) / 256), BH), 256, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_causal_prefix(const PrefixParams &p, int BH, cudaStream_t st) {
    if (p.P <= 0) return cudaSuccess;
    k_causal_prefix_features<<<dim3((p.P + 31) / 32, BH), 256, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_causal_prefix_attn<<<dim3((p.P + 63) / 64, BH), 256, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_causal_out(const CUtensorMap &mQ, const CUtensorMap &mK, const CUtensorMap &mW,
                              const CausalParams &p, int BH, cudaStream_t st) {
    const dim3 grid(p.n_split, BH);
    if (p.d != 64) return cudaErrorInvalidValue;
    const size_t sm = causal_smem<64>();
    cudaFuncSetAttribute(k_causal_out<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_causal_out<64><<<grid, kCausalThreads, sm, st>>>(mQ, mK, mW, p);
    return cudaGetLastError();
}

}  // namespace favor
