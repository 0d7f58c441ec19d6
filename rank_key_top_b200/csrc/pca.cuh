// Offline calibration of P on the GPU (AQUA page, appendix on SVD: the basis
// whose leading columns carry the most variance; Fig. 2: P is calibrated once,
// on calibration keys): for every head, the eigenvectors of the centred
// covariance of n sample keys, as the columns of P in descending eigenvalue
// order.
//
// One CTA of 512 threads per head, everything in shared memory:
//  1. covariance: C = (1/n) sum_t x_t^T x_t - mu^T mu, accumulated in fp32
//     from 64-token slabs staged in shared memory; thread t owns a 4 x 8
//     block of C;
//  2. eigendecomposition: cyclic Jacobi with the round-robin ordering, 64
//     disjoint rotations per round (d - 1 rounds a sweep), each round one
//     pass over rows and one over columns of C and of the eigenvector
//     matrix V; sweeps until every off-diagonal entry is below 2^-22 of the
//     largest diagonal entry (at most kPcaSweeps);
//  3. eigenvalues sorted descending (ties to the lower index), each column's
//     sign fixed so that its entry of largest magnitude is positive.
#pragma once

#include "common.cuh"

namespace loki {

constexpr int kPcaThreads = 512;
constexpr int kPcaSlab = 64;    // tokens staged per step of the covariance
constexpr int kPcaSweeps = 16;  // upper bound on Jacobi sweeps

struct PcaParams {
    const void* keys;  // [heads][n][D], cache type
    float* P;          // [heads][D][D]
    float* eigvals;    // [heads][D], nullable
    int64_t n;
};

template <int D>
constexpr int pca_smem_bytes() {
    return 2 * D * D * 4 + 3 * D * 4 + kPcaSlab * D * 4 + 64;  // C, V, mu/lambda/order, slab, scratch
}

template <typename T, int D>
__global__ void __launch_bounds__(kPcaThreads) pca_kernel(const PcaParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    float* C = reinterpret_cast<float*>(smem);  // [D][D]
    float* V = C + D * D;                       // [D][D]
    float* mu = V + D * D;                      // [D]
    float* lam = mu + D;                        // [D]
    int* order = reinterpret_cast<int*>(lam + D);  // [D]
    float* slab = reinterpret_cast<float*>(order + D);  // [kPcaSlab][D]
    float* scratch = slab + kPcaSlab * D;       // a few words
    const int head = blockIdx.x;
    const int tid = threadIdx.x;
    const T* x = reinterpret_cast<const T*>(p.keys) + (int64_t)head * p.n * D;

    // ---- 1. covariance ----
    // thread tid owns rows i0 .. i0 + 3 and columns j0 .. j0 + 7 of C
    constexpr int CB = D / 8;  // column blocks
    const int i0 = (tid / CB) * 4, j0 = (tid % CB) * 8;
    const bool owner = i0 < D;  // D = 128: all 512 threads; D = 64: 128 of them
    float acc[4][8];
    float msum = 0.f;  // column sum of column tid (tid < D)
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
    for (int64_t t0 = 0; t0 < p.n; t0 += kPcaSlab) {
        const int rows = p.n - t0 < kPcaSlab ? (int)(p.n - t0) : kPcaSlab;
        __syncthreads();
        for (int e = tid; e < rows * D; e += kPcaThreads) slab[e] = Elem<T>::to_f(x[(t0 * D) + e]);
        __syncthreads();
        if (tid < D)
            for (int r = 0; r < rows; ++r) msum += slab[r * D + tid];
        if (owner) {
            for (int r = 0; r < rows; ++r) {
                const float* row = slab + r * D;
                float xi[4], xj[8];
#pragma unroll
                for (int a = 0; a < 4; ++a) xi[a] = row[i0 + a];
#pragma unroll
                for (int b = 0; b < 8; ++b) xj[b] = row[j0 + b];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(xi[a], xj[b], acc[a][b]);
            }
        }
    }
    const float inv_n = 1.f / (float)p.n;
    if (tid < D) mu[tid] = msum * inv_n;
    __syncthreads();
    if (owner) {
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 8; ++b)
                C[(i0 + a) * D + j0 + b] = acc[a][b] * inv_n - mu[i0 + a] * mu[j0 + b];
    }
    for (int e = tid; e < D * D; e += kPcaThreads) V[e] = (e / D == e % D) ? 1.f : 0.f;
    __syncthreads();
    // symmetrise (the two halves were summed in different orders)
    for (int e = tid; e < D * D; e += kPcaThreads) {
        const int i = e / D, j = e % D;
        if (i < j) {
            const float v = 0.5f * (C[i * D + j] + C[j * D + i]);
            C[i * D + j] = v;
            C[j * D + i] = v;
        }
    }
    __syncthreads();

    // ---- 2. cyclic Jacobi, round-robin pairs ----
    // round r pairs position k with position D - 1 - k; position 0 holds
    // index 0, position i >= 1 holds index 1 + (i - 1 + r) mod (D - 1)
    __shared__ float cs[D / 2], sn[D / 2];
    __shared__ int pp[D / 2], pq[D / 2];
    auto at = [&](int pos, int r) { return pos == 0 ? 0 : 1 + (pos - 1 + r) % (D - 1); };
    for (int sweep = 0; sweep < kPcaSweeps; ++sweep) {
        // stop when every off-diagonal entry is negligible against the diagonal
        if (tid == 0) {
            scratch[0] = 0.f;
            scratch[1] = 0.f;
        }
        __syncthreads();
        float off = 0.f, dia = 0.f;
        for (int e = tid; e < D * D; e += kPcaThreads) {
            const int i = e / D, j = e % D;
            if (i != j) off = fmaxf(off, fabsf(C[e]));
            else dia = fmaxf(dia, fabsf(C[e]));
        }
        off = warp_max_xor(off, 0, 5);
        dia = warp_max_xor(dia, 0, 5);
        if ((tid & 31) == 0) {
            atomicMax(reinterpret_cast<int*>(scratch), __float_as_int(off));
            atomicMax(reinterpret_cast<int*>(scratch + 1), __float_as_int(dia));
        }
        __syncthreads();
        const bool done = scratch[0] <= 0x1p-22f * scratch[1];
        __syncthreads();  // every thread has read them before the next reset
        if (done) break;
        for (int r = 0; r < D - 1; ++r) {
            if (tid < D / 2) {
                int a = at(tid, r), b = at(D - 1 - tid, r);
                if (a > b) { const int tmp = a; a = b; b = tmp; }
                const float apq = C[a * D + b];
                float c = 1.f, s = 0.f;
                if (apq != 0.f) {
                    const float tau = (C[b * D + b] - C[a * D + a]) / (2.f * apq);
                    const float t = (tau >= 0.f ? 1.f : -1.f) / (fabsf(tau) + sqrtf(1.f + tau * tau));
                    c = rsqrtf(1.f + t * t);
                    s = t * c;
                }
                cs[tid] = c;
                sn[tid] = s;
                pp[tid] = a;
                pq[tid] = b;
            }
            __syncthreads();
            // rows: C <- J^T C
            for (int e = tid; e < (D / 2) * D; e += kPcaThreads) {
                const int k = e / D, j = e % D;
                const int a = pp[k], b = pq[k];
                const float c = cs[k], s = sn[k];
                const float xa = C[a * D + j], xb = C[b * D + j];
                C[a * D + j] = c * xa - s * xb;
                C[b * D + j] = s * xa + c * xb;
            }
            __syncthreads();
            // columns: C <- C J, V <- V J
            for (int e = tid; e < (D / 2) * D; e += kPcaThreads) {
                const int k = e / D, i = e % D;
                const int a = pp[k], b = pq[k];
                const float c = cs[k], s = sn[k];
                const float xa = C[i * D + a], xb = C[i * D + b];
                C[i * D + a] = c * xa - s * xb;
                C[i * D + b] = s * xa + c * xb;
                const float va = V[i * D + a], vb = V[i * D + b];
                V[i * D + a] = c * va - s * vb;
                V[i * D + b] = s * va + c * vb;
            }
            __syncthreads();
        }
    }

    // ---- 3. order, signs, output ----
    if (tid < D) lam[tid] = C[tid * D + tid];
    __syncthreads();
    if (tid < D) {  // rank of eigenvalue tid: larger ones, then equal ones at lower index
        const float v = lam[tid];
        int rank = 0;
        for (int j = 0; j < D; ++j) rank += (lam[j] > v) || (lam[j] == v && j < tid);
        order[rank] = tid;
    }
    __syncthreads();
    float* Pout = p.P + (int64_t)head * D * D;
    if (tid < D) {  // output column tid = eigenvector order[tid]
        const int src = order[tid];
        float big = 0.f, sgn = 1.f;
        for (int i = 0; i < D; ++i) {
            const float v = V[i * D + src];
            if (fabsf(v) > big) {
                big = fabsf(v);
                sgn = v < 0.f ? -1.f : 1.f;
            }
        }
        for (int i = 0; i < D; ++i) Pout[i * D + tid] = sgn * V[i * D + src];
        if (p.eigvals) p.eigvals[(int64_t)head * D + tid] = lam[src];
    }
}

}  // namespace loki
