// Routing variants (gist.science technical summary of PISA, section 2,
// covariance-aware routing): the spectral-norm reading of M_j = ||H_j - Hbar||_2.
// The pooled score without the covariance term needs no kernel of its own: the
// routing kernel runs with M_j = 0.
#pragma once

#include "common.cuh"

namespace pisa {

// M_j = largest singular value of A = H_j - Hbar, for one (batch, head, block)
// per CTA (grid (nb, BH), 256 threads).  G = A^T A is formed in shared memory
// (each thread an 8 x 8 tile for D = 128, 4 x 4 for D = 64), then power
// iteration on G until its Rayleigh quotient changes by less than 1e-7
// relative (at most kSpectralMaxIters steps); M_j = sqrt(lambda_max(G)).
// Dynamic smem: A [D][D] + G [D][D] + x [D] + y [D] + 16 partials, fp32.
constexpr int kSpectralThreads = 256;
constexpr int kSpectralMaxIters = 4000;

template <int D>
__global__ void __launch_bounds__(kSpectralThreads)
cov_spectral_kernel(const float* __restrict__ H, const float* __restrict__ hbar, int nb,
                    float* __restrict__ M) {
  extern __shared__ __align__(16) float sp[];
  float* A = sp;             // [D][D], row = key dimension
  float* G = A + D * D;      // [D][D]
  float* x = G + D * D;      // [D]
  float* y = x + D;          // [D]
  float* red = y + D;        // [16]
  const int j = blockIdx.x, bh = blockIdx.y;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const float* Hj = H + ((size_t)bh * nb + j) * D * D;
  const float* Hb = hbar + (size_t)bh * D * D;
  for (int e = t * 4; e < D * D; e += kSpectralThreads * 4) {
    const float4 h = *reinterpret_cast<const float4*>(Hj + e);
    const float4 b = *reinterpret_cast<const float4*>(Hb + e);
    *reinterpret_cast<float4*>(A + e) = make_float4(h.x - b.x, h.y - b.y, h.z - b.z, h.w - b.w);
  }
  __syncthreads();
  // G[a][c] = sum_r A[r][a] A[r][c]
  constexpr int TS = D / 16;  // tile side: 16 x 16 threads cover D x D
  const int a0 = (t / 16) * TS, c0 = (t % 16) * TS;
  float g[TS][TS];
#pragma unroll
  for (int p = 0; p < TS; ++p)
#pragma unroll
    for (int q = 0; q < TS; ++q) g[p][q] = 0.f;
  for (int r = 0; r < D; ++r) {
    float ra[TS], rc[TS];
#pragma unroll
    for (int p = 0; p < TS; ++p) {
      ra[p] = A[r * D + a0 + p];
      rc[p] = A[r * D + c0 + p];
    }
#pragma unroll
    for (int p = 0; p < TS; ++p)
#pragma unroll
      for (int q = 0; q < TS; ++q) g[p][q] = fmaf(ra[p], rc[q], g[p][q]);
  }
#pragma unroll
  for (int p = 0; p < TS; ++p)
#pragma unroll
    for (int q = 0; q < TS; ++q) G[(a0 + p) * D + c0 + q] = g[p][q];
  __syncthreads();
  // start vector: G applied to a fixed scrambled positive vector (generic, so
  // not orthogonal to the top eigenvector of real data), normalised; zero only
  // when A is
  for (int i = t; i < D; i += kSpectralThreads) y[i] = 0.5f + (float)(((uint32_t)i * 2654435761u) >> 16) * (1.f / 65536.f);
  __syncthreads();
  float dsum = 0.f;
  for (int i = t; i < D; i += kSpectralThreads) {
    float v = 0.f;
    for (int c = 0; c < D; ++c) v = fmaf(G[i * D + c], y[c], v);
    x[i] = v;
    dsum += v * v;
  }
  dsum = warp_sum(dsum);
  if (lane == 0) red[warp] = dsum;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kSpectralThreads / 32; ++w) tot += red[w];
  if (tot <= 0.f) {  // A == 0
    if (t == 0) M[(size_t)bh * nb + j] = 0.f;
    return;
  }
  const float inv0 = rsqrtf(tot);
  __syncthreads();  // every thread has read red[] and y[]
  for (int i = t; i < D; i += kSpectralThreads) x[i] *= inv0;
  __syncthreads();
  // power iteration: two threads per row of G (halves of the dot product)
  constexpr int HALF = D / 2;
  const int row = t >> 1, half = t & 1;
  const bool active = row < D;
  float lam = 0.f;
  for (int it = 0; it < kSpectralMaxIters; ++it) {
    float acc = 0.f;
    if (active) {
      const float* gr = G + row * D + half * HALF;
      const float* xs = x + half * HALF;
#pragma unroll 8
      for (int c = 0; c < HALF; ++c) acc = fmaf(gr[c], xs[c], acc);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    // partial sums of x.y (Rayleigh quotient) and y.y, one lane per row
    float xy = (active && half == 0) ? x[row] * acc : 0.f;
    float yy = (active && half == 0) ? acc * acc : 0.f;
    if (active && half == 0) y[row] = acc;
    xy = warp_sum(xy);
    yy = warp_sum(yy);
    if (lane == 0) {
      red[warp] = xy;
      red[8 + warp] = yy;
    }
    __syncthreads();
    float lxy = 0.f, lyy = 0.f;
#pragma unroll
    for (int w = 0; w < kSpectralThreads / 32; ++w) {
      lxy += red[w];
      lyy += red[8 + w];
    }
    const float prev = lam;
    lam = lxy;
    if (lyy <= 0.f) break;
    const float inv = rsqrtf(lyy);
    for (int i = t; i < D; i += kSpectralThreads) x[i] = y[i] * inv;
    __syncthreads();
    if (it > 0 && fabsf(lam - prev) <= 1e-7f * fabsf(lam)) break;
  }
  if (t == 0) M[(size_t)bh * nb + j] = sqrtf(fmaxf(lam, 0.f));
}

}  // namespace pisa
