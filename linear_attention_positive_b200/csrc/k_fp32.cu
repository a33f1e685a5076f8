// fp32 CUDA-core path: FAVOR+ forward and backward with every product and sum in fp32.
//
// One CTA per (batch, head) walks the sequence. It computes the per-head key stabiliser C (the
// maximum key logit), then, for the bidirectional FA-part ("Fast Attention Via Positive
// Orthogonal Random Features", codewithpapers.app/method/favor), the state S = (K')^T V,
// z = (K')^T 1_L followed by out_i = phi(q_i)^T S / phi(q_i)^T z; for the masked variant the
// same quantities as prefix sums over j <= i. The backward follows the chain rule through those
// definitions with W fixed (g_i = dO_i/den_i, s_i = -(dO_i . o_i)/den_i,
// dphi(q_i) = S g_i + z s_i, G = sum_i phi(q_i) g_i^T, h = sum_i phi(q_i) s_i,
// dv_j = G^T phi(k_j), dphi(k_j) = G v_j + h, dx = W^T (phi * dphi) - x sum(phi * dphi)).
//
// Stabilised features: phi(q_i)_r ~ exp(w_r.q_i - max_r' w_r'.q_i) (a per-row constant) and
// phi(k_j)_r ~ exp(w_r.k_j - |k_j|^2/2 - C) (a per-head constant); both constants cancel in the
// output and in every gradient. This path is latency-bound by design (a sequential walk per
// head); it carries the fp32 workloads, the bf16 path carries throughput.

#include "common.cuh"

namespace favor {

struct F32Params {
    int L, d, m;
    const float *Q, *K, *V, *W;   // [BH,L,d], [m,d]
    const float *out, *dout;      // backward inputs (fp32)
    float *O;                     // forward output
    float *dQ, *dK, *dV;          // backward outputs
    float *ws;                    // per head: S [m*d], G [m*d], qinfo [L*(d+2)]
};

constexpr int kF32Threads = 256;

__device__ __forceinline__ float block_reduce_max(float v, float *red) {
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float r = red[0];
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) r = fmaxf(r, red[i]);
    return r;
}

__device__ __forceinline__ float block_reduce_sum(float v, float *red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float r = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) r += red[i];
    return r;
}

// w_r . x for this thread's feature r (x in shared memory).
__device__ __forceinline__ float wdot(const float *__restrict__ W, int r, const float *x, int d) {
    const float *w = W + (size_t)r * d;
    float s = 0.f;
    for (int e = 0; e < d; ++e) s = fmaf(__ldg(w + e), x[e], s);
    return s;
}

// Loads row j of a [L,d] head tensor into shared memory (all threads), followed by a barrier.
__device__ __forceinline__ void load_row(float *dst, const float *src, int j, int d) {
    for (int e = threadIdx.x; e < d; e += blockDim.x) dst[e] = src[(size_t)j * d + e];
    __syncthreads();
}

// Shared layout: x[d] (key or query row), v[d], g[d], ph[m], y[m], z[m], h[m], red[32].
template <bool CAUSAL, bool BWD>
__global__ void __launch_bounds__(kF32Threads) k_f32_head(F32Params p) {
    extern __shared__ float sh[];
    const int d = p.d, m = p.m, L = p.L, tid = threadIdx.x;
    float *x = sh, *v = x + d, *g = v + d, *ph = g + d, *y = ph + m, *z = y + m, *hh = z + m, *red = hh + m;
    const int bh = blockIdx.x;
    const size_t off = (size_t)bh * L * d;
    const float *Q = p.Q + off, *K = p.K + off, *V = p.V + off;
    float *S = p.ws + (size_t)bh * (2 * (size_t)m * d + (size_t)L * (d + 2));
    float *G = S + (size_t)m * d;
    float *qinfo = G + (size_t)m * d;  // per query: g (d), s, c

    // ---- per-head key stabiliser C = max_j max_r (w_r.k_j - |k_j|^2/2)
    float cmax = -INFINITY;
    for (int j = 0; j < L; ++j) {
        load_row(x, K, j, d);
        float nrm = 0.f;
        for (int e = 0; e < d; ++e) nrm = fmaf(x[e], x[e], nrm);
        for (int r = tid; r < m; r += blockDim.x) cmax = fmaxf(cmax, wdot(p.W, r, x, d) - 0.5f * nrm);
        __syncthreads();
    }
    const float C = block_reduce_max(cmax, red);

    for (int i = tid; i < m * d; i += blockDim.x) S[i] = 0.f;
    for (int r = tid; r < m; r += blockDim.x) z[r] = 0.f;
    __syncthreads();

    // phi(k_j) for this thread's features, accumulated into the state S, z.
    auto add_key = [&](int j) {
        load_row(x, K, j, d);
        load_row(v, V, j, d);
        float nrm = 0.f;
        for (int e = 0; e < d; ++e) nrm = fmaf(x[e], x[e], nrm);
        for (int r = tid; r < m; r += blockDim.x) {
            const float pk = expf(wdot(p.W, r, x, d) - 0.5f * nrm - C);
            float *Sr = S + (size_t)r * d;
            for (int c = 0; c < d; ++c) Sr[c] = fmaf(pk, v[c], Sr[c]);
            z[r] += pk;
        }
        __syncthreads();
    };
    // phi(q_i) into ph[] (row-max stabilised); returns den = phi(q_i).z; leaves q_i in x.
    auto query_features = [&](int i) -> float {
        load_row(x, Q, i, d);
        float lmax = -INFINITY;
        for (int r = tid; r < m; r += blockDim.x) {
            const float u = wdot(p.W, r, x, d);
            ph[r] = u;
            lmax = fmaxf(lmax, u);
        }
        const float c = block_reduce_max(lmax, red);
        float dpart = 0.f;
        for (int r = tid; r < m; r += blockDim.x) {
            const float e = expf(ph[r] - c);
            ph[r] = e;
            dpart = fmaf(e, z[r], dpart);
        }
        const float den = block_reduce_sum(dpart, red);
        if (tid == 0) red[31] = c;
        __syncthreads();
        return den;
    };

    if (!BWD) {
        if (!CAUSAL)
            for (int j = 0; j < L; ++j) add_key(j);
        for (int i = 0; i < L; ++i) {
            if (CAUSAL) add_key(i);
            const float den = query_features(i);
            for (int c = tid; c < d; c += blockDim.x) {
                float num = 0.f;
                for (int r = 0; r < m; ++r) num = fmaf(ph[r], S[(size_t)r * d + c], num);
                p.O[off + (size_t)i * d + c] = num / den;
            }
            __syncthreads();
        }
        return;
    }

    // ---------------------------------------------------------------- backward
    const float *dO = p.dout + off;
    if (!CAUSAL)
        for (int j = 0; j < L; ++j) add_key(j);
    // Query pass (forward order): dq_i, and g_i, s_i, c_i saved for the G, h sums.
    for (int i = 0; i < L; ++i) {
        if (CAUSAL) add_key(i);
        const float den = query_features(i);
        const float c = red[31];
        // s_i uses out_i recomputed from the same features and state the gradient runs through
        // (a caller's output from a lower-precision forward would break the cancellation
        // sum_r phi(q)_r dphi(q)_r = 0 that the query gradient relies on).
        float sp = 0.f;
        for (int e = tid; e < d; e += blockDim.x) {
            float num = 0.f;
            for (int r = 0; r < m; ++r) num = fmaf(ph[r], S[(size_t)r * d + e], num);
            const float go = dO[(size_t)i * d + e];
            g[e] = go / den;
            sp = fmaf(go, num / den, sp);
        }
        const float s = -block_reduce_sum(sp, red) / den;
        float ysum = 0.f;
        for (int r = tid; r < m; r += blockDim.x) {
            const float *Sr = S + (size_t)r * d;
            float dphi = z[r] * s;
            for (int e = 0; e < d; ++e) dphi = fmaf(Sr[e], g[e], dphi);
            y[r] = ph[r] * dphi;
            ysum += y[r];
        }
        const float ys = block_reduce_sum(ysum, red);
        for (int e = tid; e < d; e += blockDim.x) {
            float acc = 0.f;
            for (int r = 0; r < m; ++r) acc = fmaf(y[r], __ldg(p.W + (size_t)r * d + e), acc);
            p.dQ[off + (size_t)i * d + e] = acc - x[e] * ys;
        }
        float *qi = qinfo + (size_t)i * (d + 2);
        for (int e = tid; e < d; e += blockDim.x) qi[e] = g[e];
        if (tid == 0) {
            qi[d] = s;
            qi[d + 1] = c;
        }
        __syncthreads();
    }
    // G = sum_i phi(q_i) g_i^T, h = sum_i phi(q_i) s_i (all i, or i >= j by a reverse walk).
    for (int i = tid; i < m * d; i += blockDim.x) G[i] = 0.f;
    for (int r = tid; r < m; r += blockDim.x) hh[r] = 0.f;
    __syncthreads();
    auto add_query = [&](int i) {
        load_row(x, Q, i, d);
        const float *qi = qinfo + (size_t)i * (d + 2);
        const float s = qi[d], c = qi[d + 1];
        for (int r = tid; r < m; r += blockDim.x) {
            const float pq = expf(wdot(p.W, r, x, d) - c);
            float *Gr = G + (size_t)r * d;
            for (int e = 0; e < d; ++e) Gr[e] = fmaf(pq, qi[e], Gr[e]);
            hh[r] = fmaf(pq, s, hh[r]);
        }
        __syncthreads();
    };
    if (!CAUSAL)
        for (int i = 0; i < L; ++i) add_query(i);
    for (int jj = 0; jj < L; ++jj) {
        const int j = CAUSAL ? L - 1 - jj : jj;
        if (CAUSAL) add_query(j);
        load_row(x, K, j, d);
        load_row(v, V, j, d);
        float nrm = 0.f;
        for (int e = 0; e < d; ++e) nrm = fmaf(x[e], x[e], nrm);
        float ysum = 0.f;
        for (int r = tid; r < m; r += blockDim.x) {
            const float pk = expf(wdot(p.W, r, x, d) - 0.5f * nrm - C);
            const float *Gr = G + (size_t)r * d;
            float dphi = hh[r];
            for (int e = 0; e < d; ++e) dphi = fmaf(Gr[e], v[e], dphi);
            ph[r] = pk;
            y[r] = pk * dphi;
            ysum += y[r];
        }
        const float ys = block_reduce_sum(ysum, red);
        for (int e = tid; e < d; e += blockDim.x) {
            float acc = 0.f, dv = 0.f;
            for (int r = 0; r < m; ++r) {
                acc = fmaf(y[r], __ldg(p.W + (size_t)r * d + e), acc);
                dv = fmaf(ph[r], G[(size_t)r * d + e], dv);
            }
            p.dK[off + (size_t)j * d + e] = acc - x[e] * ys;
            p.dV[off + (size_t)j * d + e] = dv;
        }
        __syncthreads();
    }
}

size_t f32_workspace_floats(int BH, int L, int d, int m) {
    return (size_t)BH * (2 * (size_t)m * d + (size_t)L * (d + 2));
}

cudaError_t launch_f32(const F32Params &p, int BH, bool causal, bool bwd, cudaStream_t st) {
    const size_t sm = (size_t)(3 * p.d + 4 * p.m + 32) * sizeof(float);
    if (causal) {
        if (bwd)
            k_f32_head<true, true><<<BH, kF32Threads, sm, st>>>(p);
        else
            k_f32_head<true, false><<<BH, kF32Threads, sm, st>>>(p);
    } else {
        if (bwd)
            k_f32_head<false, true><<<BH, kF32Threads, sm, st>>>(p);
        else
            k_f32_head<false, false><<<BH, kF32Threads, sm, st>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace favor
