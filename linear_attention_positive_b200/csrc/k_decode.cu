// Recurrent single-token step of the masked (causal) FA-part: the prefix-sum recurrence advanced
// by one token per head ("Random Features for Efficient Attention Approximation", abstract:
// masked self-attention; the recurrence S_t = S_{t-1} + phi(k_t) v_t^T, z_t = z_{t-1} + phi(k_t),
// out_t = phi(q_t)^T S_t / phi(q_t)^T z_t).
//
// Carried state of one head, fp32, with a per-feature stabiliser D_r (natural-log units):
//   S'[c][r] (d x m, feature-minor so a warp's loads of one value column are coalesced),
//   z'[r] (m), D[r] (m);   sum_j exp(u_r(k_j)) v_j[c] = exp(D_r) S'[c][r],
//                          sum_j exp(u_r(k_j))        = exp(D_r) z'[r],
// with u_r(x) = w_r.x - |x|^2/2 (the 1/sqrt(m) of phi cancels in the output). A feature with
// z'[r] = 0 is empty, so an all-zero buffer is the empty state. Each step raises D_r to the new
// key's logit when that is larger, rescaling the row by exp(D_old - D_new) <= 1, so S' and z'
// never overflow; the query weights exp(u_r(q) + D_r - max) are taken against their own maximum.
//
// One CTA per head, one thread per feature (m <= 256 threads). The value-column sums over
// features are reduced inside each warp by a halving exchange (each lane ends with D/32 consecutive columns),
// then across warps through shared memory. The step moves the head's state once in and once out:
// it is bound by HBM bandwidth on (m d + 2 m) * 8 bytes per head.

#include "common.cuh"

namespace favor {

struct DecodeParams {
    int BH, m;
    int bf16;                 // inputs bf16 (else fp32)
    const void *q, *k, *v;    // [BH][d]
    const void *W;            // [m][d]
    float *state;             // [BH][d*m + 2m]
    float *out;               // [BH][d]
};

template <int D>
__device__ __forceinline__ void load_vec(const void *src, int bf16, float *dst) {
    for (int c = threadIdx.x; c < D; c += blockDim.x)
        dst[c] = bf16 ? __uint_as_float((uint32_t)((const uint16_t *)src)[c] << 16) : ((const float *)src)[c];
}

// w_r . x with W row r read as 16-byte vectors (bf16 or fp32), x in shared memory.
template <int D>
__device__ __forceinline__ float row_dot(const void *W, int bf16, int r, const float *x) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (bf16) {
        const uint4 *w = (const uint4 *)((const uint16_t *)W + (size_t)r * D);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            const uint4 u = __ldg(w + i);
            const uint32_t p[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[j] = fmaf(__uint_as_float(p[j] << 16), x[8 * i + 2 * j], acc[j]);
                acc[j] = fmaf(__uint_as_float(p[j] & 0xFFFF0000u), x[8 * i + 2 * j + 1], acc[j]);
            }
        }
    } else {
        const float4 *w = (const float4 *)((const float *)W + (size_t)r * D);
#pragma unroll
        for (int i = 0; i < D / 4; ++i) {
            const float4 u = __ldg(w + i);
            acc[0] = fmaf(u.x, x[4 * i], acc[0]);
            acc[1] = fmaf(u.y, x[4 * i + 1], acc[1]);
            acc[2] = fmaf(u.z, x[4 * i + 2], acc[2]);
            acc[3] = fmaf(u.w, x[4 * i + 3], acc[3]);
        }
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

template <int D>
__global__ void __launch_bounds__(256) k_decode_step(DecodeParams p) {
    __shared__ float sq[D], sk[D], sv[D];
    __shared__ float part[8][D + 1];   // per-warp column sums
    __shared__ float red[8], redz[8];
    const int bh = blockIdx.x, r = threadIdx.x, warp = r >> 5, lane = r & 31;
    const int m = p.m, nw = m >> 5;
    load_vec<D>((const char *)p.q + (size_t)bh * D * (p.bf16 ? 2 : 4), p.bf16, sq);
    load_vec<D>((const char *)p.k + (size_t)bh * D * (p.bf16 ? 2 : 4), p.bf16, sk);
    load_vec<D>((const char *)p.v + (size_t)bh * D * (p.bf16 ? 2 : 4), p.bf16, sv);
    __syncthreads();
    float k2 = 0.f;
#pragma unroll 8
    for (int c = 0; c < D; ++c) k2 = fmaf(sk[c], sk[c], k2);
    const float uk = row_dot<D>(p.W, p.bf16, r, sk) - 0.5f * k2;
    const float uq = row_dot<D>(p.W, p.bf16, r, sq);

    float *S = p.state + (size_t)bh * ((size_t)D * m + 2 * m);
    float *z = S + (size_t)D * m, *Dl = z + m;
    const float z_old = z[r], D_old = Dl[r];
    const bool empty = !(z_old > 0.f);
    const float Dn = empty ? uk : fmaxf(D_old, uk);
    const float sc = empty ? 0.f : expf(D_old - Dn);
    const float a = expf(uk - Dn);
    float s[D];
#pragma unroll
    for (int c = 0; c < D; ++c) {
        s[c] = fmaf(S[(size_t)c * m + r], sc, a * sv[c]);
        S[(size_t)c * m + r] = s[c];
    }
    const float zn = fmaf(z_old, sc, a);
    z[r] = zn;
    Dl[r] = Dn;

    // query weights against their maximum over the head's features
    const float e = uq + Dn;
    float mx = e;
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    mx = red[0];
    for (int w = 1; w < nw; ++w) mx = fmaxf(mx, red[w]);
    const float pr = expf(e - mx);

    // per-warp sums over features of pr * s[c]: halving exchange, lane ends with D/32 columns
    // starting at lane * D/32
#pragma unroll
    for (int c = 0; c < D; ++c) s[c] *= pr;
#pragma unroll
    for (int o = 16, n = D; o > 0; o >>= 1, n >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = up ? s[i] : s[n / 2 + i];
            const float keep = up ? s[n / 2 + i] : s[i];
            s[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
#pragma unroll
    for (int j = 0; j < D / 32; ++j) part[warp][lane * (D / 32) + j] = s[j];
    float den = pr * zn;
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (lane == 0) redz[warp] = den;
    __syncthreads();
    float dd = 0.f;
    for (int w = 0; w < nw; ++w) dd += redz[w];
    for (int c = r; c < D; c += m) {
        float num = 0.f;
        for (int w = 0; w < nw; ++w) num += part[w][c];
        p.out[(size_t)bh * D + c] = num / dd;
    }
}

cudaError_t launch_decode_step(const DecodeParams &p, int d, cudaStream_t st) {
    if (d == 64)
        k_decode_step<64><<<p.BH, p.m, 0, st>>>(p);
    else
        k_decode_step<128><<<p.BH, p.m, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace favor
