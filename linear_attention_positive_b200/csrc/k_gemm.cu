// Split-precision tcgen05 GEMM with fused FAVOR+ epilogues: the building block of the bf16
// backward pass.
//
// The gradients of FAVOR+ are heavy-tailed (their largest entries are 50-90x their RMS), so a
// single 16-bit rounding of any operand of the feature contractions (phi(Q), phi(K), the state
// [S | z], the query-side sums [G | h], the products phi * dphi) already costs about 1e-2 x RMS
// on its own. Every such operand is therefore carried as a pair of bf16 values x = hi + lo
// (hi = bf16(x), lo = bf16(x - hi); 16 significant bits, fp32 range) and every product as
// hi*hi + lo*hi + hi*lo: three kind::f16 MMAs with fp32 accumulation in TMEM (two when one side
// is exact in bf16, as W, K, V and Q are). bf16 keeps fp32's exponent range, so no operand needs a
// power-of-two range scale.
//
// C[M x N] = sum_k A[M x k] B[k x N] per batch (blockIdx.z = batch * n_split + split), one
// 128 x BN output tile per CTA (BN <= 256 fp32 TMEM columns), K in 64-element tiles staged by TMA
// (128-byte swizzle) through a ring of shared-memory stages:
//   A K-major: [batch][M][K] rows of K (box 64 x 128); A M-major: [batch][K][M] (boxes 64 x 64)
//   B K-major: [batch][N][K] (box 64 x BN);            B N-major: [batch][K][N] (boxes 64 x 64)
// Optional constant blocks: a ones column appended to B (N-major, last 64 columns: column 0 = 1)
// or to A (K-major, last 64 K columns: column 0 = 1), the [V | 1] operand of the state sums.
// Warp roles (6 warps): 0 TMA, 1 MMA issue and TMEM allocation, 2-5 the epilogue (thread = row of
// the tile; TMEM lane quarter = warp % 4), which for the key feature map also sums |k|^2 from the
// A tiles while they stream through.

#include "common.cuh"

namespace favor {

enum GemmEpi : int {
    kEpiPhiQuery = 0,  // phi = exp(acc - rowmax) as hi/lo bf16 rows (N = m)
    kEpiPhiKey = 1,    // phi = 2^(acc log2e - |x|^2/2 log2e - kc[batch]) as hi/lo bf16 rows (N = m)
    kEpiGS = 2,        // [num | den | 0]: writes [g | s | 0] hi/lo, g = dO/den, s = -(dO . num/den)/den
    kEpiT = 3,         // t = phi * acc (phi from hi/lo rows), hi/lo rows and the row sums of t
    kEpiDX = 4,        // dx = acc - x * rowsum (x bf16 rows, rowsum fp32): fp32 rows
    kEpiF32 = 5,       // acc as fp32 rows
    kEpiPartial = 6,   // acc as fp32 rows of the split's partial tile [z][M][N]
    kEpiMask = 7,      // causal mask (column j kept for j <= row i, both within the batch): hi/lo rows
    kEpiOut = 8,       // [num | den]: out = num / den as fp32 rows
    kEpiRelu = 9,      // phi = max(acc, 0) as hi/lo rows (generalised attention, f = ReLU)
    kEpiTrigQ = 10,    // phi = [sin(acc), cos(acc)] as hi/lo rows of 2N (queries: exp(|q|^2/2) cancels)
    kEpiTrigK = 11,    // phi = exp(|k|^2/2) [sin(acc), cos(acc)] as hi/lo rows of 2N (|k|^2 from the A tiles)
};

struct GemmArgs {
    int M, N, K;              // per batch
    int n_split, kt_split;    // K split over CTAs: k-tiles per split
    int a_batched, b_batched; // 0: the operand is shared by all batches (batch coordinate 0)
    int a_ones, b_ones;       // constant ones block as the last K tile of A / last N block of B
    // epilogue
    int ld_out;               // row pitch (elements) of the epilogue's outputs
    uint16_t *out_hi, *out_lo;
    float *out_f32;
    float *rowsum;            // [batch][M][2]: two partial row sums (written by kEpiT, read by kEpiDX)
    const uint16_t *side_hi, *side_lo;  // kEpiT: phi rows; kEpiGS / kEpiDX: dO / x rows (hi only)
    int ld_side;
    const float *kc;          // kEpiPhiKey: per-batch key reference (log2 units)
    int d;                    // kEpiGS: number of value columns
    // chunked (causal) use: the M tile is one 128-token chunk of batch blockIdx.z
    int a_kofs;               // A's K coordinate starts at the tile's first row (A = a chunk's own rows)
    int b_nofs, b_kofs;       // B's N (K-major) / K (N-major) coordinate starts at the tile's first row
    int b_chunk, n_chunks;    // B's batch coordinate = batch * n_chunks + chunk (per-chunk images)
    int b_ones_k;             // constant ones block as the last K tile of a K-major B
    int a_mlocal;             // M-major A: M coordinate local to the chunk (0..127), not the token
    const float *addend;      // NULL, or fp32 rows (pitch ld_add) added to the accumulator first
    int ld_add;
    int out_rows;             // rows per batch of the outputs when they differ from M (else 0)
    const float *colbias;     // kEpiPhiQuery / kEpiPhiKey: NULL, or a per-column exponent offset
                              // (log2 units) added to the query logits / subtracted from the keys'
};

constexpr int kGemmThreads = 320;
constexpr int kGemmBK = 64;

struct GemmSmem {
    uint32_t a_bytes, b_bytes, stage_bytes;
    int stages;
};

// Epilogue staging: one 32-row x 32-column tile per epilogue warp (hi | lo bf16, or fp32), 4 KB.
constexpr uint32_t kGemmStageOut = 4096;
constexpr uint32_t kGemmSmemMax = 232448;  // dynamic shared memory per CTA on sm_100

// Stage ring (2 to 4 stages) that fits next to the constant blocks and the epilogue staging.
__host__ __device__ inline GemmSmem gemm_smem_plan(int BN, int a_parts, int b_parts, uint32_t const_bytes) {
    GemmSmem g;
    g.a_bytes = 128u * 128u;                      // 128 rows x 64 k x 2 B
    g.b_bytes = (uint32_t)BN * 128u;              // BN x 64 k x 2 B
    g.stage_bytes = a_parts * g.a_bytes + b_parts * g.b_bytes;
    const uint32_t budget = kGemmSmemMax - 1024u - 512u - 8u * kGemmStageOut - const_bytes;
    int s = (int)(budget / g.stage_bytes);
    g.stages = s < 2 ? 2 : (s > 4 ? 4 : s);
    return g;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float bf16_lo_f(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Splits 8 fp32 values into hi/lo bf16 (hi = rn(x), lo = rn(x - hi)) and stores 16 B of each.
__device__ __forceinline__ void store_split8(uint16_t *hi, uint16_t *lo, const float *x) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        h[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
        l[i] = pack_bf16x2(x[2 * i] - bf16_lo_f(h[i]), x[2 * i + 1] - bf16_hi_f(h[i]));
    }
    *(uint4 *)hi = make_uint4(h[0], h[1], h[2], h[3]);
    *(uint4 *)lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Loads 8 bf16 values (16 B) as fp32.
__device__ __forceinline__ void load_bf16x8(const uint16_t *p, float *x) {
    const uint4 w = *(const uint4 *)p;
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = bf16_lo_f(u[i]);
        x[2 * i + 1] = bf16_hi_f(u[i]);
    }
}

__host__ __device__ inline uint32_t gemm_const_bytes(const GemmArgs &p, int BN) {
    return (p.a_ones ? 128u * 128u : 0u) + (p.b_ones_k ? (uint32_t)BN * 128u : 0u);
}

// Loads accumulator columns [c0, c0 + 32) of this thread's row and adds the addend row, if any.
__device__ __forceinline__ void acc_row32(uint32_t t_row, int c0, const GemmArgs &p, size_t orow, int n0, bool valid,
                                          float (&v)[32]) {
    tmem_ld32(t_row + c0, v);
    if (p.addend != nullptr && valid) {
        const float4 *a = (const float4 *)(p.addend + orow * p.ld_add + n0 + c0);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 x = a[j];
            v[4 * j] += x.x;
            v[4 * j + 1] += x.y;
            v[4 * j + 2] += x.z;
            v[4 * j + 3] += x.w;
        }
    }
}

// Position of one output tile: tile index t over (M tiles, N tiles, batch x split), M fastest.
struct GemmTile {
    int m0, n0, mt, batch, split, kt0, nk, ab, bb, a_k0, b_k0, b_n0;
};

__device__ __forceinline__ GemmTile gemm_tile(const GemmArgs &p, int BN, int t) {
    GemmTile g;
    const int Mt = (p.M + 127) / 128, Nt = (p.N + BN - 1) / BN;
    g.mt = t % Mt;
    const int nt = (t / Mt) % Nt, z = t / (Mt * Nt);
    g.m0 = g.mt * 128;
    g.n0 = nt * BN;
    g.batch = z / p.n_split;
    g.split = z % p.n_split;
    const int kt_total = (p.K + kGemmBK - 1) / kGemmBK;
    g.kt0 = g.split * p.kt_split;
    g.nk = max(min(g.kt0 + p.kt_split, kt_total) - g.kt0, 0);
    g.ab = p.a_batched ? g.batch : 0;
    g.bb = p.b_chunk ? g.batch * p.n_chunks + g.mt : (p.b_batched ? g.batch : 0);
    g.a_k0 = p.a_kofs ? g.m0 : 0;
    g.b_k0 = p.b_kofs ? g.m0 : 0;
    g.b_n0 = p.b_nofs ? g.m0 : g.n0;
    return g;
}

__host__ __device__ inline int gemm_tiles(const GemmArgs &p, int BN, int batches) {
    return ((p.M + 127) / 128) * ((p.N + BN - 1) / BN) * batches * p.n_split;
}

// Persistent CTAs (one per SM) walk the output tiles t = blockIdx.x, + gridDim.x, ...; the
// accumulator is double-buffered in TMEM (2 x 256 columns), so the epilogue of one tile runs while
// the next tile's operands stream in and its MMAs run. Warp roles (10 warps): 0 TMA, 1 MMA issue and
// TMEM allocation, 2-9 the epilogue: warp w handles rows 32 (w % 4) .. + 31 of the tile (its TMEM
// lane quarter) and the column half (w - 2) / 4. The two halves never wait on each other: a
// row-wide statistic either is recomputed by each half from the accumulator (the query row maximum,
// the dot product of s) or is written as two partial values (the row sums of t, added by the
// consumer), so every wait in the kernel stays a bounded barrier wait.
template <bool A_MN, bool B_MN, bool A_SPLIT, bool B_SPLIT, int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
k_gemm(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mA2,
       const __grid_constant__ CUtensorMap mB, const __grid_constant__ CUtensorMap mB2,
       const __grid_constant__ CUtensorMap mO, const __grid_constant__ CUtensorMap mO2, GemmArgs p, int BN,
       int n_tiles) {
    constexpr int AP = A_SPLIT ? 2 : 1, BP = B_SPLIT ? 2 : 1;
    constexpr bool NORM = EPI == kEpiPhiKey || EPI == kEpiTrigK;
    constexpr int kEpiWarps = 8;
    const GemmSmem plan = gemm_smem_plan(BN, AP, BP, gemm_const_bytes(p, BN));
    const int STAGES = plan.stages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sStage = smem;
    uint8_t *sOnesA = sStage + (size_t)STAGES * plan.stage_bytes;  // 16 KB, used when a_ones
    uint8_t *sOnesB = sOnesA + (p.a_ones ? 128 * 128 : 0);           // BN x 128 B, used when b_ones_k
    uint8_t *sOut = sOnesB + (p.b_ones_k ? BN * 128 : 0);           // 8 x kGemmStageOut
    uint64_t *bars = (uint64_t *)(sOut + 8 * kGemmStageOut);
    uint64_t *full = bars, *empty = full + 4, *acc_full = empty + 4, *acc_empty = acc_full + 2, *drain = acc_empty + 2;
    uint32_t *tmem_slot = (uint32_t *)(drain + 1);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kt_total = (p.K + kGemmBK - 1) / kGemmBK;
    const int nb_load = p.b_ones ? BN / 64 - 1 : BN / 64;  // N-major B blocks loaded by TMA
    const int kt_ones = kt_total - 1;                      // the ones blocks' K tile (a_ones, b_ones_k)

    // Constant blocks: the B ones block of every stage, the A ones block, the K-major B ones block.
    if (p.b_ones) {
        for (int i = threadIdx.x; i < STAGES * BP * 64; i += kGemmThreads) {
            const int s = i / (BP * 64), part = (i / 64) % BP, k = i % 64;
            uint8_t *blk = sStage + (size_t)s * plan.stage_bytes + AP * plan.a_bytes + part * plan.b_bytes +
                           (size_t)(BN / 64 - 1) * 8192;
            uint4 *row = (uint4 *)(blk + k * 128);
            for (int c = 0; c < 8; ++c) row[c] = make_uint4(0, 0, 0, 0);
            // element (k, n = 0): chunk 0 ^ (k & 7); the lo part of a one is zero
            if (part == 0) *(uint16_t *)(blk + k * 128 + ((k & 7) << 4)) = 0x3F80;
        }
    }
    if (p.a_ones) {
        for (int r = threadIdx.x; r < 128; r += kGemmThreads) {
            uint4 *row = (uint4 *)(sOnesA + r * 128);
            for (int c = 0; c < 8; ++c) row[c] = make_uint4(0, 0, 0, 0);
            *(uint16_t *)(sOnesA + r * 128 + ((r & 7) << 4)) = 0x3F80;
        }
    }
    if (p.b_ones_k) {
        for (int r = threadIdx.x; r < BN; r += kGemmThreads) {
            uint4 *row = (uint4 *)(sOnesB + r * 128);
            for (int c = 0; c < 8; ++c) row[c] = make_uint4(0, 0, 0, 0);
            *(uint16_t *)(sOnesB + r * 128 + ((r & 7) << 4)) = 0x3F80;
        }
    }
    fence_async_smem();
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NORM ? 1 + kEpiWarps : 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiWarps);
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
    // Launched after the previous pass without waiting for it: everything above touched only this
    // CTA's shared and tensor memory. Every global read and write below comes after the previous
    // kernel has completed (and so, transitively, every kernel before it).
    pdl_launch_dependents();
    pdl_wait_prerequisites();

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (elect_one()) {
            prefetch_tensormap(&mA);
            prefetch_tensormap(&mB);
            if (A_SPLIT) prefetch_tensormap(&mA2);
            if (B_SPLIT) prefetch_tensormap(&mB2);
        }
        __syncwarp();
        int issued = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
            const GemmTile g = gemm_tile(p, BN, t);
            for (int i = 0; i < g.nk; ++i, ++issued) {
                const int s = issued % STAGES, kt = g.kt0 + i, k0 = kt * kGemmBK;
                if (!mbar_wait_lazy(&empty[s], ((issued / STAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
                if (elect_one()) {
                    uint8_t *st = sStage + (size_t)s * plan.stage_bytes;
                    const bool a_const = p.a_ones && kt == kt_ones;
                    const bool b_const = p.b_ones_k && kt == kt_ones;
                    const uint32_t bytes = (a_const ? 0u : AP * plan.a_bytes) +
                                           (b_const ? 0u : (B_MN ? BP * (uint32_t)nb_load * 8192u : BP * plan.b_bytes));
                    mbar_arrive_expect_tx(&full[s], bytes);
                    for (int part = 0; part < AP && !a_const; ++part) {
                        const CUtensorMap *m = part ? &mA2 : &mA;
                        uint8_t *dst = st + part * plan.a_bytes;
                        if (A_MN) {
                            const int am = p.a_mlocal ? 0 : g.m0;
                            tma_load_3d(dst, m, &full[s], am, g.a_k0 + k0, g.ab);
                            tma_load_3d(dst + 8192, m, &full[s], am + 64, g.a_k0 + k0, g.ab);
                        } else {
                            tma_load_3d(dst, m, &full[s], g.a_k0 + k0, g.m0, g.ab);
                        }
                    }
                    for (int part = 0; part < BP && !b_const; ++part) {
                        const CUtensorMap *m = part ? &mB2 : &mB;
                        uint8_t *dst = st + AP * plan.a_bytes + part * plan.b_bytes;
                        if (B_MN) {
                            for (int j = 0; j < nb_load; ++j)
                                tma_load_3d(dst + j * 8192, m, &full[s], g.b_n0 + 64 * j, g.b_k0 + k0, g.bb);
                        } else {
                            tma_load_3d(dst, m, &full[s], g.b_k0 + k0, g.b_n0, g.bb);
                        }
                    }
                }
                __syncwarp();
            }
        }
        // every issued copy has landed before the CTA can exit
        volatile int no_abort = 0;
        for (int i = max(issued - STAGES, 0); i < issued; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1, &no_abort);
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issue
        const uint32_t idesc = make_idesc(128, BN, kFmtBF16, A_MN ? 1u : 0u, B_MN ? 1u : 0u);
        // K-step of 16: K-major operands advance 32 B, MN-major operands 16 rows of 128 B
        constexpr uint32_t a_step = A_MN ? 2048 / 16 : 2, b_step = B_MN ? 2048 / 16 : 2;
        const uint32_t a_lbo = A_MN ? 8192 : 16, b_lbo = B_MN ? 8192 : 16;
        int consumed = 0, local = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++local) {
            const GemmTile g = gemm_tile(p, BN, t);
            const int b = local & 1;
            const uint32_t acc = tmem + (uint32_t)b * 256;
            // the epilogue has drained this accumulator buffer (two tiles ago)
            if (!mbar_wait_all(&acc_empty[b], ((local >> 1) & 1) ^ 1, abort_flag)) break;
            tc_fence_after();
            for (int i = 0; i < g.nk; ++i, ++consumed) {
                const int s = consumed % STAGES, kt = g.kt0 + i;
                if (!mbar_wait_all(&full[s], (consumed / STAGES) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t st = smem_u32(sStage) + (uint32_t)s * plan.stage_bytes;
                const bool a_const = p.a_ones && kt == kt_ones;
                const bool b_const = p.b_ones_k && kt == kt_ones;
                const uint32_t a_hi = a_const ? smem_u32(sOnesA) : st;
                const uint32_t a_lo = st + plan.a_bytes;
                const uint32_t b_hi = b_const ? smem_u32(sOnesB) : st + AP * plan.a_bytes, b_lo = b_hi + plan.b_bytes;
                const uint32_t acc0 = i > 0 ? 1u : 0u;
                mma_ss_x4_w(acc, make_sdesc(a_hi, a_lbo, 1024), make_sdesc(b_hi, b_lbo, 1024), idesc, acc0, a_step, b_step);
                if (A_SPLIT && !a_const)
                    mma_ss_x4_w(acc, make_sdesc(a_lo, a_lbo, 1024), make_sdesc(b_hi, b_lbo, 1024), idesc, 1u, a_step, b_step);
                if (B_SPLIT && !b_const)
                    mma_ss_x4_w(acc, make_sdesc(a_hi, a_lbo, 1024), make_sdesc(b_lo, b_lbo, 1024), idesc, 1u, a_step, b_step);
                mma_commit_w(&empty[s]);
            }
            if (!ok) break;
            mma_commit_w(&acc_full[b]);
        }
        // every MMA has completed before the TMEM is freed
        mma_commit_w(drain);
        volatile int no_abort = 0;
        mbar_wait_all(drain, 0, &no_abort);
    } else {
        // ------------------------------------------------------------------ epilogue
        const int q = warp & 3;             // TMEM lane quarter
        const int ch = (warp - 2) >> 2;     // column half
        const int r = q * 32 + lane;        // row of the tile
        const int HB = BN / 2;              // columns per half
        const int cb = ch * HB;             // first column of this half
        // Outputs leave through this warp's staging tile (its 32 rows x 32 columns) by TMA stores;
        // rows past the output's extent are clipped by the tensor map.
        uint8_t *stg = sOut + (size_t)(warp - 2) * kGemmStageOut;
        if (lane == 0) {
            prefetch_tensormap(&mO);
            prefetch_tensormap(&mO2);
        }
        auto stage_free = [&]() {
            if (lane == 0) bulk_wait_group_read<0>();
            __syncwarp();
        };
        // this row's 32 values as hi and lo bf16 at (column, row block, batch coordinate) of the output
        // staging layouts are the tensor maps' swizzles: 16-byte chunk j of row r at chunk
        // j ^ ((r >> 1) & 3) of its 64-byte row (bf16), j ^ (r & 7) of its 128-byte row (fp32)
        auto put_split = [&](const float *v, int col, int row0, int bz) {
            stage_free();
            uint8_t *h = stg + lane * 64, *l = stg + 2048 + lane * 64;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t off = (uint32_t)(j ^ ((lane >> 1) & 3)) << 4;
                store_split8((uint16_t *)(h + off), (uint16_t *)(l + off), v + 8 * j);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_3d(&mO, stg, col, row0, bz);
                tma_store_3d(&mO2, stg + 2048, col, row0, bz);
                bulk_commit_group();
            }
        };
        auto put_f32 = [&](const float *v, int col, int row0, int bz) {
            stage_free();
            uint8_t *o = stg + lane * 128;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *(float4 *)(o + ((j ^ (lane & 7)) << 4)) = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_3d(&mO, stg, col, row0, bz);
                bulk_commit_group();
            }
        };
        int consumed = 0, local = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++local) {
            const GemmTile g = gemm_tile(p, BN, t);
            const int row = g.m0 + r;       // row of the output
            const bool valid = row < p.M;
            const int b = local & 1;
            const uint32_t t_row = tmem + (uint32_t)b * 256 + (((uint32_t)q * 32u) << 16);
            const int row0 = g.m0 + q * 32;  // first row of this warp's block (within the batch)
            const int bz = EPI == kEpiPartial ? g.batch * p.n_split + g.split : g.batch;  // output batch
            bool ok = true;
            float sq = 0.f;                 // |x|^2 of this row (key feature map)
            if (NORM) {
                // A K-major: row r of each A tile, 8 chunks of 16 B; the whole K range is in this tile
                for (int i = 0; i < g.nk; ++i, ++consumed) {
                    const int s = consumed % STAGES;
                    if (!mbar_wait_all(&full[s], (consumed / STAGES) & 1, abort_flag)) { ok = false; break; }
                    const uint8_t *tile = sStage + (size_t)s * plan.stage_bytes;
                    float acc4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        float x[8];
                        load_bf16x8((const uint16_t *)(tile + sw128_offset(r, c)), x);
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc4[e & 3] = fmaf(x[e], x[e], acc4[e & 3]);
                    }
                    sq += (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[s]);
                }
            }
            if (!ok) break;
            if (g.nk == 0) {
                // an empty split contributes zeros (kEpiPartial only; nothing was accumulated)
                if (EPI == kEpiPartial) {
                    float z[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) z[e] = 0.f;
                    for (int c0 = cb; c0 < cb + HB; c0 += 32) put_f32(z, g.n0 + c0, row0, bz);
                }
                if (!mbar_wait_all(&acc_full[b], (local >> 1) & 1, abort_flag)) break;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[b]);
                continue;
            }
            if (!mbar_wait_all(&acc_full[b], (local >> 1) & 1, abort_flag)) break;
            tc_fence_after();
            const size_t orow = (size_t)g.batch * (p.out_rows > 0 ? p.out_rows : p.M) + row;  // output row
            if (EPI == kEpiPhiQuery || EPI == kEpiPhiKey) {
                // logit in log2 units: acc log2e (+ column offset for queries, - for keys)
                const float csign = EPI == kEpiPhiQuery ? 1.f : -1.f;
                auto col_off = [&](int c) { return p.colbias != nullptr ? csign * p.colbias[g.n0 + c] : 0.f; };
                float shift;
                if (EPI == kEpiPhiQuery) {
                    float mx = -INFINITY;  // over the whole row (both halves read it)
                    for (int c0 = 0; c0 < BN; c0 += 32) {
                        float v[32];
                        tmem_ld32(t_row + c0, v);
#pragma unroll
                        for (int e = 0; e < 32; ++e) mx = fmaxf(mx, fmaf(v[e], kLog2e, col_off(c0 + e)));
                    }
                    shift = mx;
                } else {
                    shift = 0.5f * sq * kLog2e + (p.kc != nullptr ? p.kc[g.batch] : 0.f);
                }
                for (int c0 = cb; c0 < cb + HB; c0 += 32) {
                    float v[32];
                    tmem_ld32(t_row + c0, v);
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = exp2f(fmaf(v[e], kLog2e, col_off(c0 + e) - shift));
                    put_split(v, g.n0 + c0, row0, bz);
                }
            } else if (EPI == kEpiRelu) {
                for (int c0 = cb; c0 < cb + HB; c0 += 32) {
                    float v[32];
                    tmem_ld32(t_row + c0, v);
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = fmaxf(v[e], 0.f);
                    put_split(v, g.n0 + c0, row0, bz);
                }
            } else if (EPI == kEpiTrigQ || EPI == kEpiTrigK) {
                // columns [0, N) of the row hold sin, [N, 2N) cos, of the same projections
                const float scale = EPI == kEpiTrigK ? exp2f(0.5f * sq * kLog2e) : 1.f;
                for (int c0 = cb; c0 < cb + HB; c0 += 32) {
                    float v[32], c[32];
                    tmem_ld32(t_row + c0, v);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        float sn, cs;
                        sincosf(v[e], &sn, &cs);
                        v[e] = sn * scale;
                        c[e] = cs * scale;
                    }
                    put_split(v, g.n0 + c0, row0, bz);
                    put_split(c, g.n0 + c0 + p.N, row0, bz);
                }
            } else if (EPI == kEpiGS) {
                // acc columns: num [0, d), den at d. Output [g | s | 0 ...] over BN columns.
                float den = tmem_ld1(t_row + p.d);
                if (p.addend != nullptr && valid) den += p.addend[orow * p.ld_add + p.d];
                const float inv = 1.0f / den;
                // the half that writes s (column d) takes the dot product over all d columns; the
                // other half only forms g over its own columns
                const bool owns_s = p.d >= cb && p.d < cb + HB;
                float dot = 0.f;
                const uint16_t *dO = p.side_hi + orow * p.ld_side;
                for (int c0 = owns_s ? 0 : cb; c0 < min(cb + HB, p.d); c0 += 32) {
                    float v[32], gg[32];
                    acc_row32(t_row, c0, p, orow, 0, valid, v);
                    if (valid) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) load_bf16x8(dO + c0 + 8 * j, &gg[8 * j]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) gg[e] = 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        dot = fmaf(gg[e], v[e] * inv, dot);
                        gg[e] *= inv;
                    }
                    if (c0 >= cb) put_split(gg, c0, row0, bz);
                }
                {
                    const float sv = -dot * inv;
                    for (int c0 = max(cb, p.d); c0 < cb + HB; c0 += 32) {
                        float z[32];
#pragma unroll
                        for (int e = 0; e < 32; ++e) z[e] = 0.f;
                        if (c0 == p.d) z[0] = sv;
                        put_split(z, c0, row0, bz);
                    }
                }
            } else if (EPI == kEpiOut) {
                const float inv = 1.0f / tmem_ld1(t_row + p.d);
                for (int c0 = cb; c0 < min(cb + HB, p.d); c0 += 32) {
                    float v[32];
                    tmem_ld32(t_row + c0, v);
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] *= inv;
                    put_f32(v, c0, row0, bz);
                }
            } else if (EPI == kEpiT) {
                float tsum = 0.f;
                const uint16_t *ph = p.side_hi + orow * p.ld_side + g.n0, *pl = p.side_lo + orow * p.ld_side + g.n0;
                for (int c0 = cb; c0 < cb + HB; c0 += 32) {
                    float v[32];
                    acc_row32(t_row, c0, p, orow, g.n0, valid, v);
                    if (valid) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            float h[8], l[8];
                            load_bf16x8(ph + c0 + 8 * j, h);
                            load_bf16x8(pl + c0 + 8 * j, l);
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                v[8 * j + e] *= h[e] + l[e];
                                tsum += v[8 * j + e];
                            }
                        }
                    }
                    put_split(v, g.n0 + c0, row0, bz);
                }
                if (valid) p.rowsum[2 * orow + ch] = tsum;  // two partial sums per row
            } else if (EPI == kEpiDX) {
                const float ts = valid ? p.rowsum[2 * orow] + p.rowsum[2 * orow + 1] : 0.f;
                const uint16_t *x = p.side_hi + orow * p.ld_side + g.n0;
                for (int c0 = cb; c0 < cb + HB; c0 += 32) {
                    float v[32];
                    acc_row32(t_row, c0, p, orow, g.n0, valid, v);
                    if (valid) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            float xv[8];
                            load_bf16x8(x + c0 + 8 * j, xv);
#pragma unroll
                            for (int e = 0; e < 8; ++e) v[8 * j + e] = fmaf(-xv[e], ts, v[8 * j + e]);
                        }
                    }
                    put_f32(v, g.n0 + c0, row0, bz);
                }
            } else if (EPI == kEpiMask) {
                // row = query index, column = key index (the chunk's own keys when b_nofs)
                const int col0 = p.b_nofs ? g.m0 : g.n0;
                for (int c0 = cb; c0 < cb + HB; c0 += 32) {
                    float v[32];
                    tmem_ld32(t_row + c0, v);
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (col0 + c0 + e > row) v[e] = 0.f;
                    put_split(v, g.n0 + c0, row0, bz);
                }
            } else {
                // kEpiF32 (rows of batch) and kEpiPartial (rows of batch * n_split + split)
                for (int c0 = cb; c0 < cb + HB; c0 += 32) {
                    float v[32];
                    acc_row32(t_row, c0, p, orow, g.n0, valid, v);
                    put_f32(v, g.n0 + c0, row0, bz);
                }
            }
            // this warp has read its part of the accumulator buffer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
        }
        // every bulk store of this warp has completed before the CTA exits
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// Sums the n_split partial tiles of each batch ([batch][split][M][Np] fp32, M = m features,
// columns = values | z-or-h | zero padding) in split order and writes the hi/lo bf16 image
// transposed: [batch][Np][m] (row n holds column n of every feature), the layout both the K-major
// and the N-major reads of the image expect. Block (32, 8) per 64 features x 32 columns: partial
// rows are read along n (coalesced), transposed through shared memory, written along the features.
__global__ void __launch_bounds__(256) k_gemm_reduce_image(const float *__restrict__ part, int n_split, int m, int Np,
                                                           uint16_t *img_hi, uint16_t *img_lo) {
    __shared__ float tile[64][33];
    const int batch = blockIdx.z, n_base = blockIdx.x * 32, r_base = blockIdx.y * 64;
    const int tx = threadIdx.x, ty = threadIdx.y;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int r = r_base + ty + 8 * j;
        float acc = 0.f;
        for (int s = 0; s < n_split; ++s) acc += part[(((size_t)batch * n_split + s) * m + r) * Np + n_base + tx];
        tile[ty + 8 * j][tx] = acc;
    }
    __syncthreads();
    // thread (tx, ty): columns n_base + ty + 8 i (i < 4), features r_base + 2 tx, + 1
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int nl = ty + 8 * i;
        const float a = tile[2 * tx][nl], b = tile[2 * tx + 1][nl];
        const uint32_t h = pack_bf16x2(a, b);
        const uint32_t l = pack_bf16x2(a - bf16_lo_f(h), b - bf16_hi_f(h));
        const size_t o = ((size_t)batch * Np + n_base + nl) * m + r_base + 2 * tx;
        *(uint32_t *)(img_hi + o) = h;
        *(uint32_t *)(img_lo + o) = l;
    }
}

// Sums the n_split partial tiles of each batch ([batch * n_split + s][M][Np] fp32) in split order
// into [batch][M][Np] fp32. One thread per element.
__global__ void __launch_bounds__(256) k_gemm_sum_partials(const float *__restrict__ part, int n_split, size_t per_batch,
                                                           float *__restrict__ out) {
    const size_t i = (size_t)blockIdx.x * 256 + threadIdx.x;
    if (i >= per_batch) return;
    const size_t b = blockIdx.y;
    float acc = 0.f;
    for (int s = 0; s < n_split; ++s) acc += part[(b * n_split + s) * per_batch + i];
    out[b * per_batch + i] = acc;
}

// Per-feature exponent offsets of the sequence-parallel path, log2 units:
// c_r = (|w_r|^2 / 2 - kSpKeyHeadroom) log2e. Since u_r(k) = w_r.k - |k|^2/2 <= |w_r|^2 / 2 for every
// key, 2^(u_r log2e - c_r) <= e^kSpKeyHeadroom: no key feature can overflow, and the offsets depend
// on W alone, so every rank's partial state is on the same scale.
constexpr float kSpKeyHeadroom = 40.f;

__global__ void k_feature_offsets(const uint16_t *__restrict__ W, int m, int d, float *__restrict__ c) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= m) return;
    float acc = 0.f;
    for (int e = 0; e < d; ++e) {
        const float w = __uint_as_float((uint32_t)W[(size_t)r * d + e] << 16);
        acc = fmaf(w, w, acc);
    }
    c[r] = (0.5f * acc - kSpKeyHeadroom) * kLog2e;
}

// Exclusive prefix (forward) or suffix (reverse) over the n_chunks per-chunk partial states of
// each batch ([batch * n_chunks + c][m][Np] fp32), summed in chunk order, written as hi/lo bf16
// images [batch * n_chunks + c][Np][m] (the layout of k_gemm_reduce_image). Block (32, 8) per
// 64 features x 32 columns, walking the chunks.
__global__ void __launch_bounds__(256) k_gemm_scan_image(const float *__restrict__ part, int n_chunks, int m, int Np,
                                                         int reverse, uint16_t *img_hi, uint16_t *img_lo) {
    __shared__ float tile[64][33];
    const int batch = blockIdx.z, n_base = blockIdx.x * 32, r_base = blockIdx.y * 64;
    const int tx = threadIdx.x, ty = threadIdx.y;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < n_chunks; ++i) {
        const int c = reverse ? n_chunks - 1 - i : i;
        const size_t cb = (size_t)batch * n_chunks + c;
        float val[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            tile[ty + 8 * j][tx] = acc[j];
            val[j] = part[(cb * m + r_base + ty + 8 * j) * Np + n_base + tx];
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int nl = ty + 8 * k;
            const float a = tile[2 * tx][nl], b = tile[2 * tx + 1][nl];
            const uint32_t h = pack_bf16x2(a, b);
            const uint32_t l = pack_bf16x2(a - bf16_lo_f(h), b - bf16_hi_f(h));
            const size_t o = (cb * Np + n_base + nl) * m + r_base + 2 * tx;
            *(uint32_t *)(img_hi + o) = h;
            *(uint32_t *)(img_lo + o) = l;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] += val[j];
    }
}

// ------------------------------------------------------------------------------------ host side

// Output tensor map of an epilogue: [batches][rows][ld] (bf16 or fp32) written from 32 x 32 x 1
// staging boxes with 64-byte (bf16) or 128-byte (fp32) rows, in the matching swizzle.
typedef CUresult (*GemmEncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static bool gemm_out_map(CUtensorMap *map, const void *base, bool f32, int ld, int rows, int batches) {
    static GemmEncodeFn fn = nullptr;
    if (fn == nullptr) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = (GemmEncodeFn)ptr;
    }
    if (base == nullptr) return false;
    const cuuint64_t es = f32 ? 4 : 2;
    const cuuint64_t dims[3] = {(cuuint64_t)ld, (cuuint64_t)rows, (cuuint64_t)batches};
    const cuuint64_t strides[2] = {(cuuint64_t)ld * es, (cuuint64_t)ld * rows * es};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool A_MN, bool B_MN, bool A_SPLIT, bool B_SPLIT, int EPI>
static cudaError_t launch_gemm_t(const CUtensorMap &mA, const CUtensorMap &mA2, const CUtensorMap &mB,
                                 const CUtensorMap &mB2, const GemmArgs &p, int BN, int batches, cudaStream_t st) {
    const uint32_t cb = gemm_const_bytes(p, BN);
    const GemmSmem plan = gemm_smem_plan(BN, A_SPLIT ? 2 : 1, B_SPLIT ? 2 : 1, cb);
    const size_t smem = 1024 + (size_t)plan.stages * plan.stage_bytes + cb + 8 * kGemmStageOut + 512;
    // outputs: a row block past M would be written unless M fills its tiles or the output ends at M
    const int rows = p.out_rows > 0 ? p.out_rows : p.M;
    if (rows != p.M && p.M % 128 != 0) return cudaErrorInvalidValue;
    constexpr bool F32OUT = EPI == kEpiDX || EPI == kEpiF32 || EPI == kEpiPartial || EPI == kEpiOut;
    const int zb = EPI == kEpiPartial ? batches * p.n_split : batches;
    CUtensorMap mO, mO2;
    if (F32OUT) {
        if (!gemm_out_map(&mO, p.out_f32, true, p.ld_out, rows, zb)) return cudaErrorInvalidValue;
        mO2 = mO;
    } else if (!gemm_out_map(&mO, p.out_hi, false, p.ld_out, rows, zb) ||
               !gemm_out_map(&mO2, p.out_lo, false, p.ld_out, rows, zb)) {
        return cudaErrorInvalidValue;
    }
    auto kern = k_gemm<A_MN, B_MN, A_SPLIT, B_SPLIT, EPI>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int tiles = gemm_tiles(p, BN, batches);
    const dim3 grid(std::max(1, std::min(tiles, num_sms())));
    return launch_after_previous(kern, grid, dim3(kGemmThreads), smem, st, mA, mA2, mB, mB2, mO, mO2, p, BN, tiles);
}

cudaError_t launch_scan_image(const float *part, int n_chunks, int m, int Np, int reverse, uint16_t *hi, uint16_t *lo,
                              int batches, cudaStream_t st) {
    k_gemm_scan_image<<<dim3(Np / 32, m / 64, batches), dim3(32, 8), 0, st>>>(part, n_chunks, m, Np, reverse, hi, lo);
    return cudaGetLastError();
}

cudaError_t launch_sum_partials(const float *part, int n_split, size_t per_batch, float *out, int batches,
                               cudaStream_t st) {
    k_gemm_sum_partials<<<dim3((unsigned)((per_batch + 255) / 256), batches), 256, 0, st>>>(part, n_split, per_batch, out);
    return cudaGetLastError();
}

cudaError_t launch_feature_offsets(const void *W, int m, int d, float *c, cudaStream_t st) {
    k_feature_offsets<<<(m + 127) / 128, 128, 0, st>>>((const uint16_t *)W, m, d, c);
    return cudaGetLastError();
}

cudaError_t launch_reduce_image(const float *part, int n_split, int m, int Np, uint16_t *hi, uint16_t *lo, int batches,
                                cudaStream_t st) {
    k_gemm_reduce_image<<<dim3(Np / 32, m / 64, batches), dim3(32, 8), 0, st>>>(part, n_split, m, Np, hi, lo);
    return cudaGetLastError();
}

}  // namespace favor
