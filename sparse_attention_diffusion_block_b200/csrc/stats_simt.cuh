// Block statistics, Hbar reduction and covariance norms: CUDA-core (SIMT)
// kernels used for fp32 inputs and as the reference layout of the outputs.
//
// gist.science technical summary of PISA, section 2, hardware implementation
// ("precompute": block centroids, value sums and the global statistic Hbar)
// and covariance-aware routing (M_j = ||H_j - Hbar||).
#pragma once

#include "common.cuh"

namespace pisa {

// Tile of n <= B rows x D columns of a [L, D] tensor, converted to fp32 into
// shared memory with a padded row stride D + 4 (float4-aligned, spreads banks).
template <typename T, int D>
__device__ __forceinline__ void load_rows_f32(const T* src, int n, float* dst, int B) {
  constexpr int S = D + 4;
  constexpr int V = D / 8;  // 8-element groups per row
  for (int g = threadIdx.x; g < B * V; g += blockDim.x) {
    const int r = g / V, c = (g % V) * 8;
    float x[8];
    if (r < n) {
      load8(src + (size_t)r * D + c, x);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = 0.f;
    }
    float4* o = reinterpret_cast<float4*>(dst + r * S + c);
    o[0] = make_float4(x[0], x[1], x[2], x[3]);
    o[1] = make_float4(x[4], x[5], x[6], x[7]);
  }
}

// Column sums of an fp32 smem tile [B][D+4] (rows >= n are zero).  256 threads.
template <int D>
__device__ __forceinline__ void column_sums(const float* tile, int B, float* out, float* scratch) {
  constexpr int S = D + 4;
  constexpr int G = 256 / D;  // row groups
  const int c = threadIdx.x % D, g = threadIdx.x / D;
  float acc = 0.f;
  for (int r = g; r < B; r += G) acc += tile[r * S + c];
  scratch[threadIdx.x] = acc;
  __syncthreads();
  if (threadIdx.x < D) {
    float t = 0.f;
    for (int gg = 0; gg < G; ++gg) t += scratch[gg * D + threadIdx.x];
    out[threadIdx.x] = t;
  }
  __syncthreads();
}

// acc[TA][TB] += sum_r K[r][a] * V[r][b] over the tile (a, b in this thread's
// 16x16-grid cell).  256 threads.
template <int D>
__device__ __forceinline__ void ktv_accumulate(const float* Ks, const float* Vs, int n,
                                               float (&acc)[D / 16][D / 16]) {
  constexpr int S = D + 4, T = D / 16;
  const int a0 = (threadIdx.x / 16) * T, b0 = (threadIdx.x % 16) * T;
  for (int r = 0; r < n; ++r) {
    float ka[T], vb[T];
#pragma unroll
    for (int e = 0; e < T; e += 4) {
      float4 x = *reinterpret_cast<const float4*>(Ks + r * S + a0 + e);
      float4 y = *reinterpret_cast<const float4*>(Vs + r * S + b0 + e);
      ka[e] = x.x; ka[e + 1] = x.y; ka[e + 2] = x.z; ka[e + 3] = x.w;
      vb[e] = y.x; vb[e + 1] = y.y; vb[e + 2] = y.z; vb[e + 3] = y.w;
    }
#pragma unroll
    for (int a = 0; a < T; ++a)
#pragma unroll
      for (int b = 0; b < T; ++b) acc[a][b] = fmaf(ka[a], vb[b], acc[a][b]);
  }
}

// Stats over a chunk of J consecutive blocks per CTA.  Grid (n_chunks, BH),
// 256 threads.  Writes qbar/kbar/vsum for every block and the chunk's partial
// sum_j (K_j^T V_j - kbar_j^T vsum_j) = sum_j H_j (fixed order within the chunk).
template <typename T, int D>
__global__ void __launch_bounds__(256)
stats_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  int L, int B, int nb, int J, float* __restrict__ qbar,
                  float* __restrict__ kbar, float* __restrict__ vsum, float* __restrict__ partial) {
  extern __shared__ __align__(16) float sm[];
  constexpr int S = D + 4, TT = D / 16;
  float* Ks = sm;
  float* Vs = Ks + B * S;
  float* kb = Vs + B * S;
  float* vs = kb + D;
  float* scratch = vs + D;  // 256 floats
  const int bh = blockIdx.y, chunk = blockIdx.x;
  const size_t base = (size_t)bh * L * D;
  float acc[TT][TT];
#pragma unroll
  for (int a = 0; a < TT; ++a)
#pragma unroll
    for (int b = 0; b < TT; ++b) acc[a][b] = 0.f;

  const int j_end = min(nb, (chunk + 1) * J);
  for (int j = chunk * J; j < j_end; ++j) {
    const int row0 = j * B, n = min(B, L - row0);
    // query block mean (routing only): reuse the K buffer for Q first
    load_rows_f32<T, D>(q + base + (size_t)row0 * D, n, Ks, B);
    __syncthreads();
    column_sums<D>(Ks, B, kb, scratch);
    if (threadIdx.x < D) qbar[((size_t)bh * nb + j) * D + threadIdx.x] = kb[threadIdx.x] / (float)n;
    __syncthreads();
    load_rows_f32<T, D>(k + base + (size_t)row0 * D, n, Ks, B);
    load_rows_f32<T, D>(v + base + (size_t)row0 * D, n, Vs, B);
    __syncthreads();
    column_sums<D>(Ks, B, kb, scratch);
    column_sums<D>(Vs, B, vs, scratch);
    if (threadIdx.x < D) {
      kb[threadIdx.x] = kb[threadIdx.x] / (float)n;
      kbar[((size_t)bh * nb + j) * D + threadIdx.x] = kb[threadIdx.x];
      vsum[((size_t)bh * nb + j) * D + threadIdx.x] = vs[threadIdx.x];
    }
    __syncthreads();
    ktv_accumulate<D>(Ks, Vs, n, acc);
    const int a0 = (threadIdx.x / 16) * TT, b0 = (threadIdx.x % 16) * TT;
#pragma unroll
    for (int a = 0; a < TT; ++a)
#pragma unroll
      for (int b = 0; b < TT; ++b) acc[a][b] = fmaf(-kb[a0 + a], vs[b0 + b], acc[a][b]);
    __syncthreads();
  }
  float* out = partial + ((size_t)bh * gridDim.x + chunk) * D * D;
  const int a0 = (threadIdx.x / 16) * TT, b0 = (threadIdx.x % 16) * TT;
#pragma unroll
  for (int a = 0; a < TT; ++a)
#pragma unroll
    for (int b = 0; b < TT; b += 4)
      *reinterpret_cast<float4*>(out + (a0 + a) * D + b0 + b) =
          make_float4(acc[a][b], acc[a][b + 1], acc[a][b + 2], acc[a][b + 3]);
}

// Hbar = (sum over chunks, in chunk order) / nb.  Grid (ceil(D*D/256), BH).
template <int D>
__global__ void hbar_reduce_kernel(const float* __restrict__ partial, int n_chunks, int nb,
                                   float* __restrict__ hbar) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= D * D) return;
  const float* p = partial + (size_t)bh * n_chunks * D * D + e;
  float t = 0.f;
  for (int c = 0; c < n_chunks; ++c) t += p[(size_t)c * D * D];
  hbar[(size_t)bh * D * D + e] = t / (float)nb;
}

// Per block: H_j = K_j^T V_j - kbar_j^T vsum_j.  WRITE_H: store H_j;
// otherwise M_j = ||H_j - Hbar||_F.  Grid (nb, BH), 256 threads.
template <typename T, int D, bool WRITE_H>
__global__ void __launch_bounds__(256)
block_h_simt_kernel(const T* __restrict__ k, const T* __restrict__ v, int L, int B, int nb,
                    const float* __restrict__ kbar, const float* __restrict__ vsum,
                    const float* __restrict__ hbar, float* __restrict__ out) {
  extern __shared__ __align__(16) float sm[];
  constexpr int S = D + 4, TT = D / 16;
  float* Ks = sm;
  float* Vs = Ks + B * S;
  float* red = Vs + B * S;
  const int bh = blockIdx.y, j = blockIdx.x;
  const int row0 = j * B, n = min(B, L - row0);
  const size_t base = (size_t)bh * L * D;
  load_rows_f32<T, D>(k + base + (size_t)row0 * D, n, Ks, B);
  load_rows_f32<T, D>(v + base + (size_t)row0 * D, n, Vs, B);
  __syncthreads();
  float acc[TT][TT];
#pragma unroll
  for (int a = 0; a < TT; ++a)
#pragma unroll
    for (int b = 0; b < TT; ++b) acc[a][b] = 0.f;
  ktv_accumulate<D>(Ks, Vs, n, acc);
  const int a0 = (threadIdx.x / 16) * TT, b0 = (threadIdx.x % 16) * TT;
  const float* kb = kbar + ((size_t)bh * nb + j) * D;
  const float* vs = vsum + ((size_t)bh * nb + j) * D;
  if (WRITE_H) {
    float* o = out + ((size_t)bh * nb + j) * D * D;
#pragma unroll
    for (int a = 0; a < TT; ++a)
#pragma unroll
      for (int b = 0; b < TT; ++b) o[(a0 + a) * D + b0 + b] = fmaf(-kb[a0 + a], vs[b0 + b], acc[a][b]);
  } else {
    const float* hb = hbar + (size_t)bh * D * D;
    float ss = 0.f;
#pragma unroll
    for (int a = 0; a < TT; ++a)
#pragma unroll
      for (int b = 0; b < TT; ++b) {
        const float h = fmaf(-kb[a0 + a], vs[b0 + b], acc[a][b]) - hb[(a0 + a) * D + b0 + b];
        ss = fmaf(h, h, ss);
      }
    const float tot = block_sum(ss, red);
    if (threadIdx.x == 0) out[(size_t)bh * nb + j] = sqrtf(tot);
  }
}

}  // namespace pisa
