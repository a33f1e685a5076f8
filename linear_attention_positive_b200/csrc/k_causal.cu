// Causal (masked, j <= i) FAVOR+ forward on the bf16 tensor-core path.
//
// The masked FA-part ("Random Features for Efficient Attention Approximation", thesis abstract:
// masked self-attention; the FA-part of "Fast Attention Via Positive Orthogonal Random Features",
// codewithpapers.app/method/favor, with prefix sums in place of the full sums):
//   out_i = phi(q_i)^T S_i / phi(q_i)^T z_i,   S_i = sum_{j<=i} phi(k_j) v_j^T,  z_i = sum_{j<=i} phi(k_j).
//
// Sequence parallelism: the sequence of each head is cut into segments (runs of 128-token
// tiles). k_key_partials_wide (its causal instantiation, k_keys_wide.cu) gives each segment's
// aggregate [S | z] and the per-key -|k|^2/2; k_segment_scan turns them into exclusive prefixes at
// the head's key reference C; k_causal_chunk walks each segment's tiles in order from that prefix:
//   out_tile = ( phi(Q_t) S_<t + mask(phi(Q_t) phi(K_t)^T) V_t ) / ( phi(Q_t) z_<t + rowsum(mask(...)) ),
//   S_<t+1 = S_<t + phi(K_t)^T V_t.
// The first tokens of every head are recomputed afterwards at split precision (bf16 hi + lo
// operands, k_gemm.cu): there the output is a weighted mean of few values, its magnitude is far
// above the RMS of a long output, and the 11-bit fp16 operands alone would use up the error budget.

#include "common.cuh"

namespace favor {

// ============================================================================ k_causal_chunk
//
// The chunked scan over 128-token tiles, on fp16 operands with fp32 accumulation. The m features
// are split over a cluster of m/128 CTAs (one SM each): CTA rank r owns features
// [128 r, 128 r + 128), its own fp32 running state S_r (features x 64 values, in TMEM) and z_r,
// and produces a partial output per query row; the partials are combined through distributed
// shared memory. Per tile t of a segment (tokens j0 .. j0 + 127), in CTA rank r:
//   P    = Q_t W_r^T                       (bf16 MMA; queries on TMEM lanes)
//   phiq = 2^(P log2e - c_i), c_i its row maximum over the CTA's features, fp16 into TMEM;
//          den_q = phiq . z_<t on CUDA cores
//   P^T  = W_r K_t^T                       (bf16 MMA; features on TMEM lanes)
//   phik = 2^(P^T log2e + beta_j), beta_j = (-|k_j|^2/2 - C) log2e + A, fp16 into shared memory
//          as [feature][token] rows; z_<t+1 = z_<t + sum_j phik
//   Simg = fp16(S_<t 2^-sigma_t)           (converted from TMEM; S_<t of a segment's first tile
//          is the prefix the scan wrote)
//   O    = phiq Simg                       (fp16 MMA, A from TMEM)
//   A    = phiq phik^T                     (fp16 MMA) -> masked (key > query -> 0), row sums
//          den_a = sum_j A_ij in fp32, fp16(A 2^-sigma_t) in place
//   S   += phik^T V_t                      (fp16 MMA, V_t converted bf16 -> fp16 in place)
//   O   += A V_t
//   partial numerator O 2^sigma_t, partial denominator den_q + den_a, both relative to 2^c_i.
// C is the per-(batch, head) key maximum, so phik <= 2^A with A = 8 (fp16 headroom for keys far
// below the maximum); every product phik v carries the same 2^A, which cancels in the ratio.
// sigma_t keeps the scaled S below 2^15, and with phik <= 2^8 over 128 features the scaled scores
// stay below 2^15 too. V enters as fp16 scaled by 2^-b per segment (b = max(0, e - 14), e the
// exponent of the segment's largest |v|, recorded by the key pass); the numerator is scaled back by
// 2^b with 2^sigma_t. Non-finite entries are reported as FAVOR_ERR_UNSUPPORTED through the device
// status word.
// Warp roles (16 warps): 0-3 query exponentials and den_q; 4-7 key exponentials, z and the state
// image; 8-11 masking and the output epilogue (one tile behind); 12 TMA and the key terms beta_j;
// 13 projection MMAs; 14 scores, state term, state update and masked A V MMAs; 15 V conversion.
// TMEM columns: P [0,128), phiq [128,192), A [192,320) (fp16 in [192,256)), S [320,384),
// O [384 + 64 b, +64) for b = tile parity.

struct ChunkParams {
    int L, m, n_split, tiles_per_split, P_exact;
    int n_seg;                 // BH * n_split
    const float *bias;         // [BH, L]: -|k_j|^2/2
    const float *head_max;     // [BH]: C
    const float *seg_S;        // [BH, n_split, 64, m]: exclusive prefix of S per segment, times 2^A
    const float *seg_z;        // [BH, n_split, m]: the same for z
    const uint32_t *seg_vmax;  // [BH, n_split]: the segment's largest |v| (bf16 bits)
    float *out;                // fp32 [BH, L, 64]
};

constexpr int kChunkThreads = 512;

// Power-of-two shift b of a segment's values (V' = V 2^-b in fp16): 0 while its largest |v| is
// below 2^15, else enough to bring it there; the output numerator is scaled back by 2^b.
__device__ __forceinline__ int segment_value_shift(uint32_t vmax_bits) {
    return max(0, (int)(vmax_bits >> 7) - 127 - 14);
}
constexpr float kChunkKeyShift = 8.f;

namespace chunk {
constexpr uint32_t TILE = 16384;                                // 128 rows x 128 bytes
constexpr int STAGES = 2;
constexpr uint32_t OFF_W = 0;                                   // W rows of the CTA's features
constexpr uint32_t OFF_QK = TILE;                               // stage s: Q | K
constexpr uint32_t OFF_V = OFF_QK + STAGES * 2 * TILE;          // stage s: V (fp16 after conversion)
constexpr uint32_t OFF_PHIK = OFF_V + STAGES * TILE;            // [token block][feature][64 tokens]
constexpr uint32_t OFF_SIMG = OFF_PHIK + 2 * TILE;              // [feature][64 values]
constexpr int RECV_ROW = 68;                                    // floats: numerator, den, c, pad
constexpr uint32_t RECV_SLOT = 64 * RECV_ROW * 4;               // 64 rows (two warps' bulk copies)
constexpr uint32_t OFF_RECV = OFF_SIMG + TILE;                  // [2 slots][64 rows]
constexpr uint32_t OFF_SEND = OFF_RECV + 2 * RECV_SLOT;         // staging of the rows sent
constexpr uint32_t OFF_F = OFF_SEND + RECV_SLOT;                // float arrays (indices below)
constexpr int F_ZSNAP = 0, F_BETA = 256, F_DENQ = 512, F_DENA = 768, F_CQ = 1024;  // [2][128] each
constexpr int F_SIGMA = 1280, F_SIGE = 1282, F_AMAX = 1288, F_END = 1296;
constexpr uint32_t OFF_BAR = OFF_F + F_END * 4;
enum {
    B_FULL_QK = 0, B_EMPTY_QK = 2, B_FULL_V = 4, B_EMPTY_V = 6, B_CONV = 8, B_BETA_FULL = 10, B_BETA_FREE = 12,
    B_W = 14, B_PQ_FULL, B_PK_FULL, B_PQ_FREE, B_PK_FREE, B_Z_FULL,
    B_PHIQ_FULL = B_Z_FULL + 2, B_PHIQ_FREE, B_PHIK_FULL, B_PHIK_FREE, B_S_READY, B_S_DONE, B_SIG_FULL,
    B_SC_FULL = B_SIG_FULL + 2, B_MASK_DONE, B_O_FULL, B_O_EMPTY = B_O_FULL + 2, B_DEN_FULL = B_O_EMPTY + 2,
    B_RECV_FULL = B_DEN_FULL + 2, B_RECV_FREE = B_RECV_FULL + 2, B_AMAX = B_RECV_FREE + 2, B_DRAIN = B_AMAX + 2,
    N_BAR = B_DRAIN + 2
};
constexpr uint32_t BYTES = OFF_BAR + N_BAR * 8 + 16;
constexpr uint32_t T_P = 0, T_PHIQ = 128, T_A = 192, T_S = 320, T_O = 384;
}  // namespace chunk

// The tiles one cluster walks: segments cid, cid + n_cl, ..., each its run of 128-token tiles.
struct ChunkSteps {
    int seg, tile, t1, bh, n_cl, nt;
    bool ok, first;
    __device__ void enter(const ChunkParams &p) {
        for (; seg < p.n_seg; seg += n_cl) {
            bh = seg / p.n_split;
            tile = (seg % p.n_split) * p.tiles_per_split;
            t1 = min(tile + p.tiles_per_split, nt);
            if (tile < t1) { ok = first = true; return; }
        }
        ok = false;
    }
    __device__ ChunkSteps(const ChunkParams &p, int cid, int n_cl_) : seg(cid), n_cl(n_cl_) {
        nt = (p.L + kTile - 1) / kTile;
        enter(p);
    }
    __device__ void next(const ChunkParams &p) {
        first = false;
        if (++tile == t1) {
            seg += n_cl;
            enter(p);
        }
    }
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}
// Arrive (release, cluster scope) on an mbarrier in another CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// mbar_wait_all for a barrier that another CTA of the cluster arrives on (acquire at cluster
// scope, so that the other CTA's stores before its arrive are visible).
__device__ __forceinline__ bool mbar_wait_cluster_all(uint64_t *bar, uint32_t parity, volatile int *abort) {
    const uint32_t a = smem_u32(bar);
    bool ok = mbar_try_wait_cluster(a, parity);
    if (!ok) {
        const unsigned long long t0 = globaltimer_ns();
        for (uint32_t it = 1;; ++it) {
            if (mbar_try_wait_cluster(a, parity)) { ok = true; break; }
            if ((it & 63u) == 0) {
                if (*abort) break;
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    record_status(FAVOR_ERR_TIMEOUT);
                    *abort = 1;
                    break;
                }
            }
        }
    }
    return __all_sync(0xffffffffu, ok);
}


// Bulk copy of `bytes` from this CTA's shared memory into another CTA of the cluster (destination
// and its mbarrier as cluster addresses); completes as transaction bytes on that mbarrier.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t mbar) {
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "r"(src), "r"(bytes), "r"(mbar)
                 : "memory");
}

// Shared-memory descriptors as their low 32 bits (start address and LBO fields; the high word, SBO
// = 1024 with the sm_100 version and 128-byte swizzle, is the same for every operand here), so the
// issuing warp keeps one register per operand.
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ uint32_t desc_lo(uint32_t smem_addr, uint32_t lbo_bytes) {
    return ((smem_addr >> 4) & 0x3FFFu) | (((lbo_bytes >> 4) & 0x3FFFu) << 16);
}
// D (+)= sum over 4 K-steps of A_k B_k, A and B in shared memory (low descriptor words advancing by
// a_step / b_step 16-byte units per step). Warp-collective: issued by the elect.sync lane.
__device__ __forceinline__ void mma_ss4_w(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc, uint32_t acc,
                                          uint32_t a_step, uint32_t b_step) {
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\t.reg .b32 al, bl;\n\t.reg .b64 ad, bd;\n\t"
        "setp.ne.b32 p, %4, 0;\n\tsetp.eq.b32 t, %4, %4;\n\t" FAVOR_ELECT
        "mov.b64 ad, {%1, %7};\n\tmov.b64 bd, {%2, %7};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, p;\n\t"
        "add.u32 al, %1, %5;\n\tadd.u32 bl, %2, %6;\n\tmov.b64 ad, {al, %7};\n\tmov.b64 bd, {bl, %7};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, t;\n\t"
        "add.u32 al, al, %5;\n\tadd.u32 bl, bl, %6;\n\tmov.b64 ad, {al, %7};\n\tmov.b64 bd, {bl, %7};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, t;\n\t"
        "add.u32 al, al, %5;\n\tadd.u32 bl, bl, %6;\n\tmov.b64 ad, {al, %7};\n\tmov.b64 bd, {bl, %7};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, t;\n\t}" ::"r"(d),
        "r"(a), "r"(b), "r"(idesc), "r"(acc), "r"(a_step), "r"(b_step), "r"(kDescHi)
        : "memory");
}
// The same with A in TMEM (8 columns per K-step).
__device__ __forceinline__ void mma_ts4_w(uint32_t d, uint32_t a_tmem, uint32_t b, uint32_t idesc, uint32_t acc,
                                          uint32_t b_step) {
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\t.reg .b32 al, bl;\n\t.reg .b64 bd;\n\t"
        "setp.ne.b32 p, %4, 0;\n\tsetp.eq.b32 t, %4, %4;\n\t" FAVOR_ELECT
        "mov.b64 bd, {%2, %6};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %3, p;\n\t"
        "add.u32 al, %1, 8;\n\tadd.u32 bl, %2, %5;\n\tmov.b64 bd, {bl, %6};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [al], bd, %3, t;\n\t"
        "add.u32 al, al, 8;\n\tadd.u32 bl, bl, %5;\n\tmov.b64 bd, {bl, %6};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [al], bd, %3, t;\n\t"
        "add.u32 al, al, 8;\n\tadd.u32 bl, bl, %5;\n\tmov.b64 bd, {bl, %6};\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [al], bd, %3, t;\n\t}" ::"r"(d),
        "r"(a_tmem), "r"(b), "r"(idesc), "r"(acc), "r"(b_step), "r"(kDescHi)
        : "memory");
}

// 1/x to about one ulp (MUFU; no slow-path subroutine around the epilogue's registers).
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float pow2i(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

template <int CL, int POLY>
__global__ void __launch_bounds__(kChunkThreads, 1)
k_causal_chunk(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
               const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapW, ChunkParams p) {
    using namespace chunk;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    float *sf = (float *)(smem + OFF_F);
    uint64_t *bar = (uint64_t *)(smem + OFF_BAR);
    uint32_t *tmem_slot = (uint32_t *)(bar + N_BAR);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = CL > 1 ? cluster_rank() : 0u;
    const int cid = blockIdx.x / CL, n_cl = gridDim.x / CL;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&bar[B_FULL_QK + s], 1);
            mbar_init(&bar[B_EMPTY_QK + s], 1);
            mbar_init(&bar[B_FULL_V + s], 1);
            mbar_init(&bar[B_EMPTY_V + s], 1);
            mbar_init(&bar[B_CONV + s], 32);
        }
        mbar_init(&bar[B_W], 1);
        mbar_init(&bar[B_PQ_FULL], 1);
        mbar_init(&bar[B_PK_FULL], 1);
        mbar_init(&bar[B_PQ_FREE], 128);
        mbar_init(&bar[B_PK_FREE], 128);
        mbar_init(&bar[B_PHIQ_FULL], 128);
        mbar_init(&bar[B_PHIQ_FREE], 1);
        mbar_init(&bar[B_PHIK_FULL], 128);
        mbar_init(&bar[B_PHIK_FREE], 1);
        mbar_init(&bar[B_S_READY], 128);
        mbar_init(&bar[B_S_DONE], 1);
        mbar_init(&bar[B_SC_FULL], 1);
        mbar_init(&bar[B_MASK_DONE], 128);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar[B_BETA_FULL + b], 32);
            mbar_init(&bar[B_BETA_FREE + b], 128);
            mbar_init(&bar[B_Z_FULL + b], 128);
            mbar_init(&bar[B_SIG_FULL + b], 128);
            mbar_init(&bar[B_O_FULL + b], 1);
            mbar_init(&bar[B_O_EMPTY + b], 128);
            mbar_init(&bar[B_DEN_FULL + b], 256);
            mbar_init(&bar[B_RECV_FULL + b], 1);
            mbar_init(&bar[B_RECV_FREE + b], 64);
            mbar_init(&bar[B_AMAX + b], 4);
        }
        mbar_init(&bar[B_DRAIN], 1);
        mbar_init(&bar[B_DRAIN + 1], 1);
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
    if (CL > 1) cluster_sync_all();  // the partner's barriers exist before any remote arrive or copy
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_off = ((uint32_t)(warp & 3) * 32u) << 16;
    const int row = (warp & 3) * 32 + lane;  // TMEM lane of this thread (query row or feature)

    if (warp >= 12) {
        regs_dec<72>();
        if (warp == 12) {
            // ---- TMA: W once; Q, K of tile g and V of tile g - 1 per step (V is needed later and
            // its stage is held until the tile's last MMA); the key terms
            // beta_j = (-|k_j|^2/2 - C) log2e + A of tile g (4 tokens per lane)
            if (elect_one()) {
                prefetch_tensormap(&mapQ);
                prefetch_tensormap(&mapK);
                prefetch_tensormap(&mapV);
                prefetch_tensormap(&mapW);
                mbar_arrive_expect_tx(&bar[B_W], TILE);
                tma_load_2d(smem + OFF_W, &mapW, &bar[B_W], 0, 128 * (int)rank);
            }
            __syncwarp();
            int g = 0, pbh = 0, ptile = 0;
            bool ok = true;
            for (ChunkSteps it(p, cid, n_cl);; ++g) {
                const bool have = it.ok;
                if (have) {
                    const int s = g % STAGES, b = g & 1;
                    if (!(ok = mbar_wait_lazy(&bar[B_EMPTY_QK + s], ((g / STAGES) & 1) ^ 1, abort_flag))) break;
                    if (elect_one()) {
                        uint8_t *st = smem + OFF_QK + s * 2 * TILE;
                        mbar_arrive_expect_tx(&bar[B_FULL_QK + s], 2 * TILE);
                        tma_load_3d(st, &mapQ, &bar[B_FULL_QK + s], 0, it.tile * kTile, it.bh);
                        tma_load_3d(st + TILE, &mapK, &bar[B_FULL_QK + s], 0, it.tile * kTile, it.bh);
                    }
                    __syncwarp();
                    if (g >= 2 && !(ok = mbar_wait_all(&bar[B_BETA_FREE + b], ((g >> 1) - 1) & 1, abort_flag))) break;
                    const float cb = kChunkKeyShift - p.head_max[it.bh] * kLog2e;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int jt = lane * 4 + k, j = it.tile * kTile + jt;
                        sf[F_BETA + b * 128 + jt] =
                            j < p.L ? fmaf(p.bias[(size_t)it.bh * p.L + j], kLog2e, cb) : -INFINITY;
                    }
                    mbar_arrive(&bar[B_BETA_FULL + b]);
                }
                if (g > 0) {
                    const int e = g - 1, s = e % STAGES;
                    if (!(ok = mbar_wait_lazy(&bar[B_EMPTY_V + s], ((e / STAGES) & 1) ^ 1, abort_flag))) break;
                    if (elect_one()) {
                        mbar_arrive_expect_tx(&bar[B_FULL_V + s], TILE);
                        tma_load_3d(smem + OFF_V + s * TILE, &mapV, &bar[B_FULL_V + s], 0, ptile * kTile, pbh);
                    }
                    __syncwarp();
                }
                if (!have) break;
                pbh = it.bh;
                ptile = it.tile;
                it.next(p);
            }
            // wait for the copies in flight (bounded) before the CTA may exit
            volatile int no_abort = 0;
            const int nq = ok ? g : g + 1;  // Q/K copies issued
            for (int i = max(nq - STAGES, 0); i < nq; ++i)
                mbar_wait(&bar[B_FULL_QK + i % STAGES], (i / STAGES) & 1, &no_abort);
            const int nv = ok ? g : max(g - 1, 0);
            for (int i = max(nv - STAGES, 0); i < nv; ++i)
                mbar_wait(&bar[B_FULL_V + i % STAGES], (i / STAGES) & 1, &no_abort);
            mbar_wait(&bar[B_W], 0, &no_abort);
        } else if (warp == 13 || warp == 14) {
            // ---- MMA issue in two independent streams (each thread's commits track its own MMAs):
            // warp 13 the projections into P (Q W^T, W K^T), warp 14 everything that produces the
            // output and the state (scores, state term, state update, masked A V')
            const uint32_t id_proj = make_idesc(128, 128, kFmtBF16, 0, 0);
            const uint32_t id_64 = make_idesc(128, 64, kFmtF16, 0, 1);
            const uint32_t id_sc = make_idesc(128, 128, kFmtF16, 0, 1);
            const uint32_t base = smem_u32(smem);
            constexpr uint32_t kTileU = TILE / 16, kRow16 = 2048 / 16, kHalfU = 8192 / 16;
            int n = 0;
            for (ChunkSteps it(p, cid, n_cl); it.ok; it.next(p)) ++n;
            bool ok = true;
            if (warp == 13) {
                // K-major operands (LBO unused)
                const uint32_t dW = desc_lo(base + OFF_W, 16);
                const uint32_t dQK = desc_lo(base + OFF_QK, 16);
                ok = mbar_wait_all(&bar[B_W], 0, abort_flag);
                if (ok && n > 0) {
                    ok = mbar_wait_all(&bar[B_FULL_QK], 0, abort_flag);
                    tc_fence_after();
                    if (ok) {
                        mma_ss4_w(tmem + T_P, dQK, dW, id_proj, 0u, 2, 2);
                        mma_commit_w(&bar[B_PQ_FULL]);
                    }
                }
                for (int g = 0; ok && g < n; ++g) {
                    const int s = g % STAGES;
                    const uint32_t ph = g & 1;
                    // K projection of tile g, once the query warps have read P; frees the Q/K stage
                    if (!(ok = mbar_wait_all(&bar[B_PQ_FREE], ph, abort_flag))) break;
                    tc_fence_after();
                    {
                        mma_ss4_w(tmem + T_P, dW, dQK + (2 * s + 1) * kTileU, id_proj, 0u, 2, 2);
                        mma_commit_w(&bar[B_PK_FULL]);
                        mma_commit_w(&bar[B_EMPTY_QK + s]);
                    }
                    // Q projection of tile g + 1, once the key warps have read P
                    if (g + 1 < n) {
                        const int s1 = (g + 1) % STAGES;
                        if (!(ok = mbar_wait_all(&bar[B_FULL_QK + s1], ((g + 1) / STAGES) & 1, abort_flag))) break;
                        if (!(ok = mbar_wait_all(&bar[B_PK_FREE], ph, abort_flag))) break;
                        tc_fence_after();
                        {
                            mma_ss4_w(tmem + T_P, dQK + 2 * s1 * kTileU, dW, id_proj, 0u, 2, 2);
                            mma_commit_w(&bar[B_PQ_FULL]);
                        }
                    }
                }
            } else {
                // MN-major operands (LBO = 16 KB between 64-wide blocks) and phik^T as K-major A
                const uint32_t dV0 = desc_lo(base + OFF_V, TILE);
                const uint32_t dKB = desc_lo(base + OFF_PHIK, TILE);
                const uint32_t dKA = desc_lo(base + OFF_PHIK, 16);
                const uint32_t dSimg = desc_lo(base + OFF_SIMG, TILE);
                // O += mask(A) V' of tile e
                auto issue_av = [&](int e) -> bool {
                    if (!mbar_wait_all(&bar[B_MASK_DONE], e & 1, abort_flag)) return false;
                    tc_fence_after();
                    {
                        const uint32_t tO = tmem + T_O + 64 * (e & 1), dV = dV0 + (e % STAGES) * kTileU;
                        mma_ts4_w(tO, tmem + T_A, dV, id_64, 1u, kRow16);
                        mma_ts4_w(tO, tmem + T_A + 32, dV + kHalfU, id_64, 1u, kRow16);
                        mma_commit_w(&bar[B_O_FULL + (e & 1)]);
                        mma_commit_w(&bar[B_EMPTY_V + e % STAGES]);
                    }
                    return true;
                };
                int g = 0;
                for (; ok && g < n; ++g) {
                    const int s = g % STAGES, b = g & 1;
                    const uint32_t ph = g & 1;
                    // the previous tile's O += mask(A) V' (before this tile's scores overwrite A)
                    if (g > 0 && !(ok = issue_av(g - 1))) break;
                    // A = phiq phik^T
                    if (!(ok = mbar_wait_all(&bar[B_PHIQ_FULL], ph, abort_flag))) break;
                    if (!(ok = mbar_wait_all(&bar[B_PHIK_FULL], ph, abort_flag))) break;
                    tc_fence_after();
                    {
                        mma_ts4_w(tmem + T_A, tmem + T_PHIQ, dKB, id_sc, 0u, kRow16);
                        mma_ts4_w(tmem + T_A, tmem + T_PHIQ + 32, dKB + kHalfU, id_sc, 1u, kRow16);
                        mma_commit_w(&bar[B_SC_FULL]);
                    }
                    // O = phiq Simg
                    if (!(ok = mbar_wait_all(&bar[B_S_READY], ph, abort_flag))) break;
                    if (g >= 2 && !(ok = mbar_wait_all(&bar[B_O_EMPTY + b], ((g >> 1) - 1) & 1, abort_flag))) break;
                    tc_fence_after();
                    {
                        const uint32_t tO = tmem + T_O + 64 * b;
                        mma_ts4_w(tO, tmem + T_PHIQ, dSimg, id_64, 0u, kRow16);
                        mma_ts4_w(tO, tmem + T_PHIQ + 32, dSimg + kHalfU, id_64, 1u, kRow16);
                        mma_commit_w(&bar[B_PHIQ_FREE]);
                    }
                    // S += phik^T V'
                    if (!(ok = mbar_wait_all(&bar[B_CONV + s], (g / STAGES) & 1, abort_flag))) break;
                    tc_fence_after();
                    {
                        const uint32_t dV = dV0 + s * kTileU;
                        mma_ss4_w(tmem + T_S, dKA, dV, id_64, 1u, 2, kRow16);
                        mma_ss4_w(tmem + T_S, dKA + kTileU, dV + kHalfU, id_64, 1u, 2, kRow16);
                        mma_commit_w(&bar[B_PHIK_FREE]);
                        mma_commit_w(&bar[B_S_DONE]);
                    }
                }
                if (ok && n > 0) issue_av(n - 1);
            }
            mma_commit_w(&bar[B_DRAIN + (warp - 13)]);
            volatile int no_abort = 0;
            mbar_wait(&bar[B_DRAIN + (warp - 13)], 0, &no_abort);
        } else {
            // ---- V tiles bf16 -> fp16 in place, times 2^-b of their segment (non-finite entries are
            // reported)
            int g = 0;
            for (ChunkSteps it(p, cid, n_cl); it.ok; it.next(p), ++g) {
                const int s = g % STAGES;
                if (!mbar_wait_lazy(&bar[B_FULL_V + s], (g / STAGES) & 1, abort_flag)) break;
                uint8_t *vt = smem + OFF_V + s * TILE;
                const float vsc = pow2i((float)-segment_value_shift(__ldg(p.seg_vmax + it.seg)));
                uint32_t mx = 0;
#pragma unroll 4
                for (int q = lane; q < (int)(TILE / 16); q += 32) {
                    uint4 *pq = (uint4 *)(vt + q * 16);
                    const uint4 w = *pq;
                    mx = __vmaxu2(mx, w.x & 0x7FFF7FFFu);
                    mx = __vmaxu2(mx, w.y & 0x7FFF7FFFu);
                    mx = __vmaxu2(mx, w.z & 0x7FFF7FFFu);
                    mx = __vmaxu2(mx, w.w & 0x7FFF7FFFu);
                    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
                    uint32_t h[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        float lo, hi;
                        ffma2(__uint_as_float(u[k] << 16), __uint_as_float(u[k] & 0xFFFF0000u), vsc, vsc, 0.f, 0.f, lo, hi);
                        h[k] = pack_f16x2(lo, hi);
                    }
                    *pq = make_uint4(h[0], h[1], h[2], h[3]);
                }
                // inf / nan entries (bf16 exponent field all ones) have no scaled fp16 form
                if (max(mx & 0xFFFFu, mx >> 16) >= 0x7F80u) record_status(FAVOR_ERR_UNSUPPORTED);
                fence_async_smem();
                mbar_arrive(&bar[B_CONV + s]);
            }
        }
    } else if (warp < 4) {
        // ---- query exponentials: thread = query row (the row of logits in registers, so P is
        // released at once)
        regs_inc<208>();
        int g = 0;
        for (ChunkSteps it(p, cid, n_cl); it.ok; it.next(p), ++g) {
            const int b = g & 1;
            float v[128];
            if (!mbar_wait_all(&bar[B_PQ_FULL], g & 1, abort_flag)) break;
            tc_fence_after();
            tmem_ld128(tmem + lane_off + T_P, v);
            tc_fence_before();
            mbar_arrive(&bar[B_PQ_FREE]);
            const float cl = row_max128(v) * kLog2e;
#pragma unroll
            for (int e = 0; e < 128; e += 2) ffma2(v[e], v[e + 1], kLog2e, kLog2e, -cl, -cl, v[e], v[e + 1]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
#pragma unroll
                for (int e = 32 * c; e < 32 * c + 32 - POLY; ++e) v[e] = ex2_approx(v[e]);
#pragma unroll
                for (int e = 32 * c + 32 - POLY; e < 32 * c + 32; e += 2) exp2_poly_pair(v[e], v[e + 1], v[e], v[e + 1]);
            }
            // den_q = phiq . z_<t (z_<t is published before the state term of tile g - 1 frees phiq)
            if (!mbar_wait_all(&bar[B_Z_FULL + b], (g >> 1) & 1, abort_flag)) break;
            const float *z = sf + F_ZSNAP + b * 128;
            float d0 = 0.f, d1 = 0.f;
#pragma unroll
            for (int e = 0; e < 128; e += 4) {
                const float4 z4 = *(const float4 *)(z + e);
                ffma2(v[e], v[e + 1], z4.x, z4.y, d0, d1, d0, d1);
                ffma2(v[e + 2], v[e + 3], z4.z, z4.w, d0, d1, d0, d1);
            }
            if (g > 0 && !mbar_wait_all(&bar[B_PHIQ_FREE], (g - 1) & 1, abort_flag)) break;
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                uint32_t hv[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) hv[e] = pack_f16x2(v[32 * h + 2 * e], v[32 * h + 2 * e + 1]);
                tmem_st16u(tmem + lane_off + T_PHIQ + 16 * h, hv);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar[B_PHIQ_FULL]);
            if (g >= 2 && !mbar_wait_all(&bar[B_O_EMPTY + b], ((g >> 1) - 1) & 1, abort_flag)) break;
            sf[F_DENQ + b * 128 + row] = d0 + d1;
            sf[F_CQ + b * 128 + row] = cl;
            mbar_arrive(&bar[B_DEN_FULL + b]);
        }
    } else if (warp < 8) {
        // ---- key exponentials, z, and the fp16 state image: thread = feature
        regs_dec<104>();
        const int f = row;
        const int fg = 128 * (int)rank + f;  // feature index within m
        float z = 0.f;
        int g = 0;
        for (ChunkSteps it(p, cid, n_cl); it.ok; it.next(p), ++g) {
            const int s = g % STAGES, b = g & 1;
            const size_t srow = (size_t)it.seg * p.m + fg;
            if (it.first) {
                // a segment starts from the scan's prefix: S master <- seg_S once the last state
                // MMA of the previous segment has completed; z_<t published for the query warps
                z = p.seg_z[srow];
                sf[F_ZSNAP + b * 128 + f] = z;
                mbar_arrive(&bar[B_Z_FULL + b]);
                if (g > 0 && !mbar_wait_all(&bar[B_S_DONE], (g - 1) & 1, abort_flag)) break;
                tc_fence_after();
                // feature-minor rows: thread f reads column c at p.seg_S[(seg * 64 + c) * m + fg]; the
                // prefix takes the segment's value scale 2^-b
                const float *src = p.seg_S + (size_t)it.seg * 64 * p.m + fg;
                const float vsc = pow2i((float)-segment_value_shift(__ldg(p.seg_vmax + it.seg)));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float w[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) w[c] = __ldg(src + (size_t)(32 * h + c) * p.m) * vsc;
                    tmem_st32(tmem + lane_off + T_S + 32 * h, w);
                }
                tmem_wait_st();
            }
            // phik = 2^(P^T log2e + beta_j) per 32-token chunk straight from TMEM (the next chunk's load
            // in flight), each chunk stored to shared memory as fp16 ([token block][feature][64 tokens])
            // once the previous tile's MMAs have read phik; P is held until the last chunk is read
            if (!mbar_wait_all(&bar[B_PK_FULL], g & 1, abort_flag)) break;
            if (!mbar_wait_all(&bar[B_BETA_FULL + b], (g >> 1) & 1, abort_flag)) break;
            if (g > 0 && !mbar_wait_all(&bar[B_PHIK_FREE], (g - 1) & 1, abort_flag)) break;
            tc_fence_after();
            const float *beta = sf + F_BETA + b * 128;
            uint8_t *pk = smem + OFF_PHIK + f * 128;
            float zs0 = 0.f, zs1 = 0.f;
            float va[32], vb[32];
            tmem_ld32(tmem + lane_off + T_P, va);
#pragma unroll 2
            for (int c = 0; c < 4; ++c) {
                float(&v)[32] = (c & 1) ? vb : va;
                float(&vn)[32] = (c & 1) ? va : vb;
                if (c < 3)
                    asm volatile(
                        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
                        "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
                        "%30, %31}, [%32];"
                        : FAVOR_REG32(vn)
                        : "r"(tmem + lane_off + T_P + 32 * (c + 1)));
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 b4 = *(const float4 *)(beta + 32 * c + e);
                    ffma2(v[e], v[e + 1], kLog2e, kLog2e, b4.x, b4.y, v[e], v[e + 1]);
                    ffma2(v[e + 2], v[e + 3], kLog2e, kLog2e, b4.z, b4.w, v[e + 2], v[e + 3]);
                }
#pragma unroll
                for (int e = 0; e < 32 - POLY; ++e) v[e] = ex2_approx(v[e]);
#pragma unroll
                for (int e = 32 - POLY; e < 32; e += 2) exp2_poly_pair(v[e], v[e + 1], v[e], v[e + 1]);
                uint32_t hv[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    ffma2(v[e], v[e + 1], 1.f, 1.f, zs0, zs1, zs0, zs1);
                    hv[e >> 1] = pack_f16x2(v[e], v[e + 1]);
                }
                // tokens 32c .. 32c + 31: block c >> 1, 16-byte chunks 4 (c & 1) .. + 3
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    *(uint4 *)(pk + (c >> 1) * TILE + (((4 * (c & 1) + u) ^ (f & 7)) << 4)) =
                        make_uint4(hv[4 * u], hv[4 * u + 1], hv[4 * u + 2], hv[4 * u + 3]);
                if (c < 3) asm volatile("tcgen05.wait::ld.sync.aligned;" : FAVOR_RW32(vn)::"memory");
            }
            tc_fence_before();
            mbar_arrive(&bar[B_PK_FREE]);
            mbar_arrive(&bar[B_BETA_FREE + b]);
            z += zs0 + zs1;
            {
                // z_<t+1 for the next tile, unless that tile starts a segment (its z is the prefix)
                ChunkSteps nx = it;
                nx.next(p);
                if (nx.ok && !nx.first) {
                    sf[F_ZSNAP + (b ^ 1) * 128 + f] = z;
                    mbar_arrive(&bar[B_Z_FULL + (b ^ 1)]);
                }
            }
            fence_async_smem();
            mbar_arrive(&bar[B_PHIK_FULL]);
            // state image of tile g from S_<g (the state MMA of tile g - 1 has completed)
            if (g > 0 && !it.first && !mbar_wait_all(&bar[B_S_DONE], (g - 1) & 1, abort_flag)) break;
            tc_fence_after();
            float amax = 0.f;
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                float w[32];
                tmem_ld32(tmem + lane_off + T_S + 32 * h, w);
#pragma unroll
                for (int c = 0; c < 32; ++c) amax = fmaxf(amax, fabsf(w[c]));
            }
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            if (lane == 0) {
                sf[F_AMAX + b * 4 + (warp & 3)] = amax;
                mbar_arrive(&bar[B_AMAX + b]);
            }
            if (!mbar_wait_all(&bar[B_AMAX + b], (g >> 1) & 1, abort_flag)) break;
            amax = fmaxf(fmaxf(sf[F_AMAX + b * 4], sf[F_AMAX + b * 4 + 1]),
                         fmaxf(sf[F_AMAX + b * 4 + 2], sf[F_AMAX + b * 4 + 3]));
            // sigma: amax 2^-sigma < 2^15
            const int ea = (int)((__float_as_uint(amax) >> 23) & 0xFFu) - 127;
            const int sig = max(ea - 14, 0);
            const float sc = pow2i(-sig);
            uint8_t *simg = smem + OFF_SIMG + f * 128;
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                float w[32];
                tmem_ld32(tmem + lane_off + T_S + 32 * h, w);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float x[8];
#pragma unroll
                    for (int i = 0; i < 8; i += 2) ffma2(w[8 * c + i], w[8 * c + i + 1], sc, sc, 0.f, 0.f, x[i], x[i + 1]);
                    uint4 u;
                    u.x = pack_f16x2(x[0], x[1]);
                    u.y = pack_f16x2(x[2], x[3]);
                    u.z = pack_f16x2(x[4], x[5]);
                    u.w = pack_f16x2(x[6], x[7]);
                    *(uint4 *)(simg + (((4 * h + c) ^ (f & 7)) << 4)) = u;
                }
            }
            if (f == 0) sf[F_SIGMA + b] = (float)sig;
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bar[B_S_READY]);
            mbar_arrive(&bar[B_SIG_FULL + b]);
        }
    } else {
        // ---- masking (tile g) and the output epilogue (tile e = g - 1): thread = query row. Per
        // step: the partial output of tile e is read from TMEM (rows the partner finishes are
        // staged and sent at once), tile g is masked, then this CTA's rows of tile e are finished
        // with the partner's half, which has arrived meanwhile.
        const int q = warp & 3;
        const bool keep = CL == 1 || (uint32_t)(row >> 6) == rank;  // warp-uniform
        const uint32_t partner = rank ^ 1u;
        ChunkSteps it(p, cid, n_cl);
        int pbh = 0, pj0 = 0;
        for (int g = 0;; ++g) {
            const bool have = it.ok;
            const int e = g - 1, eb = e & 1;
            float o[64], den = 0.f, cq = 0.f, up = 1.f;
            if (g > 0) {
                // A. tile e: partial output and denominators
                if (!mbar_wait_all(&bar[B_O_FULL + eb], (e >> 1) & 1, abort_flag)) break;
                if (!mbar_wait_all(&bar[B_DEN_FULL + eb], (e >> 1) & 1, abort_flag)) break;
                tc_fence_after();
                tmem_ld64_nowait(tmem + lane_off + T_O + 64 * eb, o);
                asm volatile("tcgen05.wait::ld.sync.aligned;" : FAVOR_RW32((&o[0])), FAVOR_RW32((&o[32]))::"memory");
                den = sf[F_DENQ + eb * 128 + row] + sf[F_DENA + eb * 128 + row];
                cq = sf[F_CQ + eb * 128 + row];
                up = pow2i((int)sf[F_SIGE + eb]);
                tc_fence_before();
                mbar_arrive(&bar[B_O_EMPTY + eb]);
                if (!keep) {
                    // rows the partner finishes: stage them, one bulk copy per warp
                    if (e >= 2 && !mbar_wait_cluster_all(&bar[B_RECV_FREE + eb], ((e >> 1) - 1) & 1, abort_flag))
                        break;
                    if (lane == 0) bulk_wait_group_read<0>();  // the previous copy has read the staging rows
                    __syncwarp();
                    float *srow = (float *)(smem + OFF_SEND) + (row & 63) * RECV_ROW;
#pragma unroll
                    for (int c = 0; c < 64; c += 4) {
                        float4 w;
                        ffma2(o[c], o[c + 1], up, up, 0.f, 0.f, w.x, w.y);
                        ffma2(o[c + 2], o[c + 3], up, up, 0.f, 0.f, w.z, w.w);
                        *(float4 *)(srow + c) = w;
                    }
                    *(float4 *)(srow + 64) = make_float4(den, cq, 0.f, 0.f);
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        const uint32_t off = (uint32_t)((row & 63) * RECV_ROW * 4);  // this warp's first row
                        bulk_copy_to_peer(cluster_map(smem_u32(smem + OFF_RECV + eb * RECV_SLOT) + off, partner),
                                          smem_u32(smem + OFF_SEND) + off, 32 * RECV_ROW * 4,
                                          cluster_map(smem_u32(&bar[B_RECV_FULL + eb]), partner));
                        bulk_commit_group();
                    }
                    __syncwarp();
                } else if (CL > 1 && row == 64 * (int)rank) {
                    // arm for the partner's two bulk copies of tile e
                    mbar_arrive_expect_tx(&bar[B_RECV_FULL + eb], 64 * RECV_ROW * 4);
                }
            }
            if (have) {
                // B. masking of tile g
                const int b = g & 1;
                if (!mbar_wait_all(&bar[B_SC_FULL], g & 1, abort_flag)) break;
                if (!mbar_wait_all(&bar[B_SIG_FULL + b], (g >> 1) & 1, abort_flag)) break;
                tc_fence_after();
                const int sig = (int)sf[F_SIGMA + b];
                const float sc = pow2i(-sig);
                float rs0 = 0.f, rs1 = 0.f;
#pragma unroll 1
                for (int k = 0; k < 4; ++k) {
                    uint32_t h[16];
                    if (k <= q) {
                        float a[32];
                        tmem_ld32(tmem + lane_off + T_A + 32 * k, a);
                        if (k == q) {
#pragma unroll
                            for (int c = 0; c < 32; ++c) a[c] = c <= lane ? a[c] : 0.f;
                        }
#pragma unroll
                        for (int c = 0; c < 32; c += 2) {
                            float s0, s1;
                            ffma2(a[c], a[c + 1], 1.f, 1.f, rs0, rs1, rs0, rs1);
                            ffma2(a[c], a[c + 1], sc, sc, 0.f, 0.f, s0, s1);
                            h[c >> 1] = pack_f16x2(s0, s1);
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 16; ++c) h[c] = 0u;
                    }
                    tmem_st16u(tmem + lane_off + T_A + 16 * k, h);
                }
                if (g >= 2 && !mbar_wait_all(&bar[B_O_EMPTY + b], ((g >> 1) - 1) & 1, abort_flag)) break;
                sf[F_DENA + b * 128 + row] = rs0 + rs1;
                // the output's scale back: 2^sigma of the scores and 2^b of the segment's values
                if (row == 0) sf[F_SIGE + b] = (float)(sig + segment_value_shift(__ldg(p.seg_vmax + it.seg)));
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bar[B_MASK_DONE]);
                mbar_arrive(&bar[B_DEN_FULL + b]);
            }
            if (g > 0 && keep) {
                // C. this CTA's rows of tile e
                const int i = pj0 + row;
                float *dst = p.out + ((size_t)pbh * p.L + i) * 64;
                const bool store = i < p.L && i >= p.P_exact;
                if (CL == 1) {
                    const float inv = up * rcp_approx(den);
                    if (store)
#pragma unroll
                        for (int c = 0; c < 64; c += 4) {
                            float4 w;
                            ffma2(o[c], o[c + 1], inv, inv, 0.f, 0.f, w.x, w.y);
                            ffma2(o[c + 2], o[c + 3], inv, inv, 0.f, 0.f, w.z, w.w);
                            *(float4 *)(dst + c) = w;
                        }
                } else {
                    if (!mbar_wait_cluster_all(&bar[B_RECV_FULL + eb], (e >> 1) & 1, abort_flag)) break;
                    const float *slot = (const float *)(smem + OFF_RECV + eb * RECV_SLOT) + (row & 63) * RECV_ROW;
                    const float4 dc = *(const float4 *)(slot + 64);
                    const float m2 = fmaxf(cq, dc.y);
                    const float wa = ex2_approx(cq - m2), wb = ex2_approx(dc.y - m2);
                    const float inv = rcp_approx(den * wa + dc.x * wb);
                    const float sa = up * wa * inv, sb = wb * inv;
#pragma unroll
                    for (int c = 0; c < 64; c += 4) {
                        const float4 r4 = *(const float4 *)(slot + c);
                        float t0, t1, t2, t3;
                        ffma2(r4.x, r4.y, sb, sb, 0.f, 0.f, t0, t1);
                        ffma2(r4.z, r4.w, sb, sb, 0.f, 0.f, t2, t3);
                        ffma2(o[c], o[c + 1], sa, sa, t0, t1, o[c], o[c + 1]);
                        ffma2(o[c + 2], o[c + 3], sa, sa, t2, t3, o[c + 2], o[c + 3]);
                    }
                    mbar_arrive_remote(cluster_map(smem_u32(&bar[B_RECV_FREE + eb]), partner));
                    if (store)
#pragma unroll
                        for (int c = 0; c < 64; c += 4) *(float4 *)(dst + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
                }
            }
            if (!have) break;
            pbh = it.bh;
            pj0 = it.tile * kTile;
            it.next(p);
        }
        // the last bulk copies have read their staging rows before the CTA may exit
        if (CL > 1 && lane == 0) bulk_wait_group_all();
    }
    tc_fence_before();
    __syncthreads();
    if (CL > 1) cluster_sync_all();  // no CTA leaves while its partner may still access its memory
    tc_fence_after();
    if (warp == 13) tmem_dealloc(tmem, 512);
}

// ============================================================================ host launchers


// The register split of k_causal_chunk (208 + 104 + 128 + 72 per warpgroup lane) fits the 128 per
// thread it is launched with; the launch is refused unless the kernel carries exactly 128.
template <int CL, int POLY>
static cudaError_t launch_causal_chunk_t(const CUtensorMap &mQ, const CUtensorMap &mK, const CUtensorMap &mV,
                                         const CUtensorMap &mW, const ChunkParams &p, cudaStream_t st) {
    static int checked = 0;
    static int n_cl = 0;
    const size_t sm = 1024 + chunk::BYTES;
    if (checked == 0) {
        cudaFuncAttributes a{};
        checked = (cudaFuncGetAttributes(&a, k_causal_chunk<CL, POLY>) == cudaSuccess && a.numRegs == 128) ? 1 : -1;
        if (checked > 0 &&
            cudaFuncSetAttribute(k_causal_chunk<CL, POLY>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) !=
                cudaSuccess)
            checked = -1;
        if (checked > 0) {
            cudaLaunchConfig_t cfg{};
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = CL;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.gridDim = dim3(CL * 1024);
            cfg.blockDim = dim3(kChunkThreads);
            cfg.dynamicSmemBytes = sm;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n_cl, k_causal_chunk<CL, POLY>, &cfg) != cudaSuccess || n_cl < 1)
                checked = -1;
        }
    }
    if (checked < 0) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(CL * std::min(n_cl, p.n_seg)));
    cfg.blockDim = dim3(kChunkThreads);
    cfg.dynamicSmemBytes = sm;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_causal_chunk<CL, POLY>, mQ, mK, mV, mW, p);
}

cudaError_t launch_causal_chunk(const CUtensorMap &mQ, const CUtensorMap &mK, const CUtensorMap &mV,
                                const CUtensorMap &mW, const ChunkParams &p, int poly_pct, cudaStream_t st) {
    const int poly = poly_pct < 13 ? 0 : poly_pct < 31 ? 8 : poly_pct < 44 ? 12 : 16;
    if (p.m == 128) {
        switch (poly) {
            case 0: return launch_causal_chunk_t<1, 0>(mQ, mK, mV, mW, p, st);
            case 8: return launch_causal_chunk_t<1, 8>(mQ, mK, mV, mW, p, st);
            case 12: return launch_causal_chunk_t<1, 12>(mQ, mK, mV, mW, p, st);
            default: return launch_causal_chunk_t<1, 16>(mQ, mK, mV, mW, p, st);
        }
    }
    if (p.m != 256) return cudaErrorInvalidValue;
    switch (poly) {
        case 0: return launch_causal_chunk_t<2, 0>(mQ, mK, mV, mW, p, st);
        case 8: return launch_causal_chunk_t<2, 8>(mQ, mK, mV, mW, p, st);
        case 12: return launch_causal_chunk_t<2, 12>(mQ, mK, mV, mW, p, st);
        default: return launch_causal_chunk_t<2, 16>(mQ, mK, mV, mW, p, st);
    }
}

}  // namespace favor
