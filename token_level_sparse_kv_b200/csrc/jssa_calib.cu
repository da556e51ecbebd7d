// Calibration of the shared query-key basis P from sampled queries and keys:
// the step before the decode path.
//
// Method: "Joint Subspace Sparse Attention for Efficient Long-Context
// Decoding", Abstract (a spectral solution for the shared low-dimensional
// query-key subspace); news item "JSSA makes token-level sparse decoding
// gather-free", Interpretation para 2 (queries and keys preserved jointly).
// The pages give no objective or closed form; the reading computed here is
// the plainest spectral one: per KV head h,
//   S_q = sum q q^T over the sampled queries of the head's G query heads,
//   S_k = sum k k^T over the sampled keys,
//   M   = S_q / tr(S_q) + S_k / tr(S_k),
//   P   = an orthonormal basis of the top-r eigenvectors of M
// (the selection score q^T P P^T k depends on P only through its span).
// Sampled keys: per batch row b, n tokens t_j = floor(j * T_b / n), j < n
// (all t < T_b when T_b <= n); sampled queries: every row of q_cal [N, Hq, d].
//
// Two kernels:
//  * calib_moment_kernel: one CTA per (KV head, chunk of samples), each
//    thread owning 8 x 8 tiles of the d x d sum, samples staged through
//    shared memory 32 at a time; the chunks' partial sums go to the
//    workspace (a fixed-order second pass keeps the result deterministic);
//  * calib_basis_kernel: one CTA per KV head adds the partials in order,
//    normalises by the traces, and runs subspace iteration from the given
//    basis, X <- orth(M X), orthonormalising with classical Gram-Schmidt
//    applied twice (one block reduction per column and pass).
#include "jssa_common.cuh"
#include "jssa_internal.h"

namespace jssa {

namespace {

constexpr int kCT = 256;     // threads
constexpr int kBatch = 32;   // sample vectors staged per round

template <typename KV>
__device__ __forceinline__ float ldf(const void *p, size_t i) {
    return to_f32(static_cast<const KV *>(p)[i]);
}

template <typename KV, int D>
__global__ void __launch_bounds__(kCT) calib_moment_kernel(CalibArgs a) {
    __shared__ float xs[kBatch][D];
    constexpr int NT8 = D / 8;                // tiles per matrix row
    constexpr int TILES = NT8 * NT8;          // 8 x 8 tiles of the d x d sum
    constexpr int PASSES = (TILES + kCT - 1) / kCT;
    const int h = blockIdx.x, chunk = blockIdx.y, tid = threadIdx.x;
    const int G = a.Hq / a.Hkv;
    const bool queries = chunk == a.chunks;   // the last chunk takes the queries
    const long long nsamp = queries ? (long long)a.Nq * G : (long long)a.B * a.n_keys;
    const long long s0 = queries ? 0 : chunk * nsamp / a.chunks;
    const long long s1 = queries ? nsamp : (chunk + 1) * nsamp / a.chunks;
    float *dst = queries ? a.Sq + (size_t)h * D * D : a.Sk + ((size_t)h * a.chunks + chunk) * D * D;

#pragma unroll 1
    for (int pass = 0; pass < PASSES; ++pass) {
        const int tile = pass * kCT + tid;
        const bool own = tile < TILES;
        const int ti = own ? tile / NT8 : 0, tj = own ? tile % NT8 : 0;
        float acc[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
        for (long long sb = s0; sb < s1; sb += kBatch) {
            const int nb = (int)min((long long)kBatch, s1 - sb);
            __syncthreads();
            for (int e = tid; e < kBatch * D; e += kCT) {
                const int v = e / D, c = e - v * D;
                float x = 0.f;
                if (v < nb) {
                    const long long s = sb + v;
                    if (queries) {
                        const long long n = s / G, g = s - n * G;
                        x = ldf<KV>(a.q, ((size_t)n * a.Hq + (size_t)h * G + g) * D + c);
                    } else {
                        const int b = (int)(s / a.n_keys), j = (int)(s - (long long)b * a.n_keys);
                        const int Tb = clamp_seq(a.seq_lens[b], a.T_cap, a.status);
                        if (Tb <= a.n_keys ? j < Tb : true) {
                            const long long t = Tb <= a.n_keys ? j : (long long)j * Tb / a.n_keys;
                            x = ldf<KV>(a.K, (((size_t)b * a.T_cap + t) * a.Hkv + h) * D + c);
                        }
                    }
                }
                xs[v][c] = x;
            }
            __syncthreads();
            if (own) {
                for (int v = 0; v < nb; ++v) {
                    float xi[8], xj[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        xi[u] = xs[v][ti * 8 + u];
                        xj[u] = xs[v][tj * 8 + u];
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i)
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(xi[i], xj[j], acc[i][j]);
                }
            }
        }
        if (own) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) dst[(size_t)(ti * 8 + i) * D + tj * 8 + j] = acc[i][j];
        }
    }
}

__device__ __forceinline__ float block_sum(float v, float *red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[w] = v;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < kCT / 32; ++i) t += red[i];
    return t;
}

// X, Y: [r][D] in shared memory (column c of the basis is row c).
template <int D>
__global__ void __launch_bounds__(kCT) calib_basis_kernel(CalibArgs a) {
    extern __shared__ float sm[];
    const int r = a.r;
    float *X = sm;                       // [r][D]
    float *Y = X + (size_t)r * D;        // [r][D]
    float *coef = Y + (size_t)r * D;     // [r]
    float *red = coef + 128;             // [kCT / 32]
    const int h = blockIdx.x, tid = threadIdx.x;
    float *M = a.M + (size_t)h * D * D;
    // M = sum of the key partials / its trace + the query sum / its trace
    float trk = 0.f, trq = 0.f;
    for (int i = tid; i < D; i += kCT) {
        trq += a.Sq[(size_t)h * D * D + (size_t)i * D + i];
        for (int c = 0; c < a.chunks; ++c) trk += a.Sk[((size_t)h * a.chunks + c) * D * D + (size_t)i * D + i];
    }
    trq = block_sum(trq, red);
    trk = block_sum(trk, red);
    const float iq = trq > 0.f ? 1.f / trq : 0.f, ik = trk > 0.f ? 1.f / trk : 0.f;
    for (int e = tid; e < D * D; e += kCT) {
        float sk = 0.f;
        for (int c = 0; c < a.chunks; ++c) sk += a.Sk[((size_t)h * a.chunks + c) * D * D + e];
        M[e] = sk * ik + a.Sq[(size_t)h * D * D + e] * iq;
    }
    for (int e = tid; e < r * D; e += kCT) {
        const int c = e / D, i = e - c * D;
        X[e] = a.P_init[((size_t)h * D + i) * r + c];
    }
    __syncthreads();
    for (int it = 0; it < a.iters; ++it) {
        // Y = M X (M symmetric: thread i reads column i of M, coalesced over i)
        for (int i = tid; i < D; i += kCT) {
            float y[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) y[c] = 0.f;
            for (int k = 0; k < D; ++k) {
                const float m = __ldcg(M + (size_t)k * D + i);
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (c < r) y[c] = fmaf(m, X[(size_t)c * D + k], y[c]);
            }
#pragma unroll
            for (int c = 0; c < 64; ++c)
                if (c < r) Y[(size_t)c * D + i] = y[c];
        }
        __syncthreads();
        // X = orth(Y): classical Gram-Schmidt, twice per column
        for (int c = 0; c < r; ++c) {
            for (int pass = 0; pass < 2; ++pass) {
                // coef[p] = X_p . Y_c for p < c: one warp per p
                const int w = tid >> 5, lane = tid & 31;
                for (int p = w; p < c; p += kCT / 32) {
                    float s = 0.f;
                    for (int i = lane; i < D; i += 32) s = fmaf(X[(size_t)p * D + i], Y[(size_t)c * D + i], s);
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
                    if (lane == 0) coef[p] = s;
                }
                __syncthreads();
                for (int i = tid; i < D; i += kCT) {
                    float v = Y[(size_t)c * D + i];
                    for (int p = 0; p < c; ++p) v = fmaf(-coef[p], X[(size_t)p * D + i], v);
                    Y[(size_t)c * D + i] = v;
                }
                __syncthreads();
            }
            float nn = 0.f;
            for (int i = tid; i < D; i += kCT) nn = fmaf(Y[(size_t)c * D + i], Y[(size_t)c * D + i], nn);
            nn = block_sum(nn, red);
            const float inv = nn > 0.f ? rsqrtf(nn) : 0.f;
            for (int i = tid; i < D; i += kCT) X[(size_t)c * D + i] = Y[(size_t)c * D + i] * inv;
            __syncthreads();
        }
    }
    for (int e = tid; e < r * D; e += kCT) {
        const int c = e / D, i = e - c * D;
        a.P_out[((size_t)h * D + i) * r + c] = X[e];
    }
}

template <typename KV>
cudaError_t launch_calib_kv(const CalibArgs &a, int d, cudaStream_t s) {
    void (*mk)(CalibArgs) = nullptr;
    void (*bk)(CalibArgs) = nullptr;
    switch (d) {
        case 64: mk = calib_moment_kernel<KV, 64>; bk = calib_basis_kernel<64>; break;
        case 128: mk = calib_moment_kernel<KV, 128>; bk = calib_basis_kernel<128>; break;
        case 256: mk = calib_moment_kernel<KV, 256>; bk = calib_basis_kernel<256>; break;
        default: return cudaErrorInvalidValue;
    }
    cudaError_t e = launch_kernel(mk, dim3(a.Hkv, a.chunks + 1), dim3(kCT), 0, s, false, a);
    if (e != cudaSuccess) return e;
    const size_t smem = ((size_t)2 * a.r * d + 128 + kCT / 32) * sizeof(float);
    return launch_kernel(bk, dim3(a.Hkv), dim3(kCT), smem, s, false, a);
}

}  // namespace

int calib_chunks(int Hkv) {
    int c = device_sm_count() / (Hkv > 0 ? Hkv : 1);
    return c < 1 ? 1 : (c > 64 ? 64 : c);
}

cudaError_t launch_calib(const CalibArgs &a, int kv_dtype, int d, cudaStream_t s) {
    if (a.r < 1 || a.r > 64) return cudaErrorInvalidValue;
    return kv_dtype == JSSA_BF16 ? launch_calib_kv<__nv_bfloat16>(a, d, s) : launch_calib_kv<float>(a, d, s);
}

}  // namespace jssa
