// Covariance-aware top-k routing (AI Radio summary of PISA: score
// Score_{t,j}; gist.science technical summary, section 2, covariance-aware
// routing).  For query block i of a (batch, head):
//   score_{i,j} = s qbar_i . kbar_j + ln(n_j + s ||qbar_i||_2 M_j)
//   sel[i]      = the k largest scores, exact ties to the smaller j, ascending.
#pragma once

#include "common.cuh"

namespace pisa {

// Order-preserving map float -> uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t orderable_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Grid (ceil(nb / R), BH), 256 threads (8 warps), dynamic smem:
//   Qb [R][D] fp32, Kc [32][D+4] fp32, keys [R][nb] uint32, qn [R], mj [32], nj [32].
// Phase 1 computes the R x nb scores with fp32 FMAs (tile of 32 key blocks at a
// time) and stores their orderable keys; phase 2 runs, per row (one warp per
// row), an MSB-first bitwise search for the k-th largest key, then writes the
// selected indices in ascending order.
template <int D>
__global__ void __launch_bounds__(256)
select_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
              const float* __restrict__ M, int L, int B, int nb, int kk, int R,
              float scale, int32_t* __restrict__ sel) {
  extern __shared__ __align__(16) float sm[];
  constexpr int KS = D + 4;
  float* Qb = sm;                              // R * D
  float* Kc = Qb + R * D;                      // 32 * KS
  float* qn = Kc + 32 * KS;                    // R
  float* mj = qn + R;                          // 32
  float* nj = mj + 32;                         // 32
  uint32_t* keys = reinterpret_cast<uint32_t*>(nj + 32);  // R * nb
  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * R;
  const int rows = min(R, nb - i0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int e = threadIdx.x; e < R * D; e += blockDim.x) {
    const int r = e / D;
    Qb[e] = (r < rows) ? qbar[((size_t)bh * nb + i0 + r) * D + (e % D)] : 0.f;
  }
  __syncthreads();
  for (int r = warp; r < R; r += 8) {
    float t = 0.f;
    for (int a = lane; a < D; a += 32) t = fmaf(Qb[r * D + a], Qb[r * D + a], t);
    t = warp_sum(t);
    if (lane == 0) qn[r] = sqrtf(t);
  }

  // Phase 1: scores.  Thread t handles key column c = t % 32 of the tile and
  // rows r = t / 32, t / 32 + 8, ...
  for (int j0 = 0; j0 < nb; j0 += 32) {
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * D; e += blockDim.x) {
      const int c = e / D, a = e % D;
      Kc[c * KS + a] = (j0 + c < nb) ? kbar[((size_t)bh * nb + j0 + c) * D + a] : 0.f;
    }
    if (threadIdx.x < 32) {
      const int j = j0 + threadIdx.x;
      mj[threadIdx.x] = (j < nb) ? M[(size_t)bh * nb + j] : 0.f;
      nj[threadIdx.x] = (j < nb) ? (float)min(B, L - j * B) : 1.f;
    }
    __syncthreads();
    const int c = lane;
    const int j = j0 + c;
    if (j < nb) {
      for (int r = warp; r < rows; r += 8) {
        float dot = 0.f;
#pragma unroll 8
        for (int a = 0; a < D; a += 4) {
          const float4 x = *reinterpret_cast<const float4*>(Qb + r * D + a);
          const float4 y = *reinterpret_cast<const float4*>(Kc + c * KS + a);
          dot = fmaf(x.x, y.x, dot);
          dot = fmaf(x.y, y.y, dot);
          dot = fmaf(x.z, y.z, dot);
          dot = fmaf(x.w, y.w, dot);
        }
        const float sc = scale * dot + logf(nj[c] + scale * qn[r] * mj[c]);
        keys[r * nb + j] = orderable_key(sc);
      }
    }
  }
  __syncthreads();

  // Phase 2: per-row selection.
  const int C = (nb + 31) / 32;  // contiguous chunk of indices per lane
  for (int r = warp; r < rows; r += 8) {
    const uint32_t* kr = keys + r * nb;
    uint32_t prefix = 0;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = prefix | (1u << bit);
      int cnt = 0;
      for (int j = lane; j < nb; j += 32) cnt += (kr[j] >= cand);
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (cnt >= kk) prefix = cand;
    }
    const uint32_t thr = prefix;  // k-th largest key
    const int jb = lane * C, je = min(nb, jb + C);
    int n_gt = 0, n_eq = 0;
    for (int j = jb; j < je; ++j) {
      n_gt += (kr[j] > thr);
      n_eq += (kr[j] == thr);
    }
    const int tot_gt = __reduce_add_sync(0xffffffffu, n_gt);
    const int need = kk - tot_gt;  // ties taken, lowest indices first
    // exclusive scans over lanes
    int eq_before = n_eq, sel_before;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, eq_before, o);
      if (lane >= o) eq_before += y;
    }
    eq_before -= n_eq;
    const int take_eq = max(0, min(n_eq, need - eq_before));
    const int mine = n_gt + take_eq;
    sel_before = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, sel_before, o);
      if (lane >= o) sel_before += y;
    }
    sel_before -= mine;
    int32_t* out = sel + ((size_t)bh * nb + i0 + r) * kk;
    int pos = sel_before, eq_taken = 0;
    for (int j = jb; j < je; ++j) {
      const uint32_t key = kr[j];
      bool take = key > thr;
      if (key == thr && eq_taken < take_eq) {
        take = true;
        ++eq_taken;
      }
      if (take) out[pos++] = j;
    }
  }
}

}  // namespace pisa
