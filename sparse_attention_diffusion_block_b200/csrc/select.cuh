// Covariance-aware top-k routing (AI Radio summary of PISA: score
// Score_{t,j}; gist.science technical summary, section 2, covariance-aware
// routing).  For query block i of a (batch, head):
//   score_{i,j} = s qbar_i . kbar_j + ln(n_j + s ||qbar_i||_2 M_j)
//   sel[i]      = the k largest scores, exact ties to the smaller j, ascending.
// With M == nullptr the covariance term drops out (M_j = 0): score =
// s qbar_i . kbar_j + ln n_j, plain pooled block-sparse routing.
#pragma once

#include "common.cuh"

namespace pisa {

// Order-preserving map float -> uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t orderable_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Count of the warp's keys kv (NR per lane) that are >= c: four independent
// partial counts, a short dependency chain to the reduce.
template <int NR>
__device__ __forceinline__ int count_at_least(const uint32_t (&kv)[NR], uint32_t c) {
  int c4[4] = {0, 0, 0, 0};
#pragma unroll
  for (int m = 0; m < NR; ++m) c4[m & 3] += (kv[m] >= c);
  return __reduce_add_sync(0xffffffffu, (c4[0] + c4[1]) + (c4[2] + c4[3]));
}

// The k largest of the nb keys kr[0..nb) (exact ties to the smaller index),
// written to out[0..k) in ascending index order.  One warp per row, every lane
// calls it.  Lane l holds keys j = l + 32 m (m < NR, nb <= 32 NR) in registers.
// A search over key values finds a threshold: a key value t with exactly k
// keys >= t (any such t separates the top k), or else the k-th largest key
// itself.  A 0 key stands for "no block" and is never counted: every
// candidate is above the smallest real key.
//   - NR >= 16: a bracket lo < hi with count(>= lo) >= k > count(>= hi); each
//     round tries the candidate that linear interpolation of the two counts
//     points to, and a round that fails to halve the bracket makes the next
//     one bisect, so the search ends within 64 rounds (~9-10 on the video
//     workloads, against ~12-17 for the bitwise search);
//   - NR < 16: MSB-first bitwise search below the common high bits of the
//     largest and smallest key (a round is cheap enough that the extra
//     interpolation arithmetic would not pay).
// Then, for m = 0, 1, ..., the warp takes the keys above the threshold and
// the first of the keys equal to it, and places them with ballots and prefix
// counts: indices come out ascending.
template <int NR>
__device__ __forceinline__ void topk_row_regs(const uint32_t* __restrict__ kr, int nb, int kk, int lane,
                                              int32_t* __restrict__ out) {
  uint32_t kv[NR];
  uint32_t mx = 0u, mn = 0xffffffffu;
#pragma unroll
  for (int m = 0; m < NR; ++m) {
    const int j = lane + 32 * m;
    kv[m] = (j < nb) ? kr[j] : 0u;
    if (j < nb) {
      mx = max(mx, kv[m]);
      mn = min(mn, kv[m]);
    }
  }
  mx = __reduce_max_sync(0xffffffffu, mx);
  mn = __reduce_min_sync(0xffffffffu, mn);
  uint32_t thr = mn;  // k == nb: every key
  if (kk < nb) {
    if constexpr (NR >= 16) {
      uint64_t lo = mn, hi = (uint64_t)mx + 1u;  // count(>= lo) = nb, count(>= hi) = 0
      int clo = nb, chi = 0;
      bool bisect = false, found = false;
      while (hi - lo > 1u) {
        const uint64_t w = hi - lo;
        uint64_t cand;
        if (bisect) {
          cand = lo + w / 2u;
        } else {
          const float f = (float)(clo - kk) / (float)(clo - chi);
          cand = lo + (uint64_t)(f * (float)w);
          cand = cand < lo + 1u ? lo + 1u : (cand > hi - 1u ? hi - 1u : cand);
        }
        const int cnt = count_at_least(kv, (uint32_t)cand);
        if (cnt == kk) {
          thr = (uint32_t)cand;
          found = true;
          break;
        }
        if (cnt > kk) {
          lo = cand;
          clo = cnt;
        } else {
          hi = cand;
          chi = cnt;
        }
        bisect = (hi - lo) > w / 2u;
      }
      if (!found) thr = (uint32_t)lo;  // the k-th largest key (ties at it)
    } else {
      // the k-th largest lies in [mn, mx], so it shares their common high bits
      thr = mx;
      const uint32_t diff = mx ^ mn;
      if (diff != 0u) {
        const int top = 31 - __clz(diff);
        uint32_t prefix = (top == 31) ? 0u : (mx & ~((2u << top) - 1u));
        for (int bit = top; bit >= 0; --bit) {
          const uint32_t cand = prefix | (1u << bit);
          const int cnt = count_at_least(kv, cand);
          if (cnt >= kk) {
            prefix = cand;
            // exactly k keys are >= cand: they are the top k, and cand
            // separates them from the rest as well as the k-th key would
            if (cnt == kk) break;
          }
        }
        thr = prefix;
      }
    }
  }
  int gt = 0;
#pragma unroll
  for (int m = 0; m < NR; ++m) gt += (kv[m] > thr);
  int need = kk - __reduce_add_sync(0xffffffffu, gt);  // ties taken, lowest indices first
  const uint32_t below = (1u << lane) - 1u;
  int base = 0;
#pragma unroll
  for (int m = 0; m < NR; ++m) {
    const bool eq = kv[m] == thr;
    const uint32_t be = __ballot_sync(0xffffffffu, eq);
    const bool take = kv[m] > thr || (eq && __popc(be & below) < need);
    const uint32_t bt = __ballot_sync(0xffffffffu, take);
    if (take) out[base + __popc(bt & below)] = lane + 32 * m;
    base += __popc(bt);
    need -= min(__popc(be), max(need, 0));
  }
}

// The same for any nb, keys read from shared memory: lane l takes the
// contiguous indices [l C, l C + C).
__device__ __forceinline__ void topk_row_smem(const uint32_t* __restrict__ kr, int nb, int kk, int lane,
                                              int32_t* __restrict__ out) {
  uint32_t prefix = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = prefix | (1u << bit);
    int cnt = 0;
    for (int j = lane; j < nb; j += 32) cnt += (kr[j] >= cand);
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= kk) {
      prefix = cand;
      if (cnt == kk) break;
    }
  }
  const uint32_t thr = prefix;
  const int C = (nb + 31) / 32;
  const int jb = min(nb, lane * C), je = min(nb, jb + C);
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

__device__ __forceinline__ void topk_row_ascending(const uint32_t* __restrict__ kr, int nb, int kk, int lane,
                                                   int32_t* __restrict__ out) {
  // as few key registers per lane as the row needs (a multiple of four)
  if (nb <= 128) {
    topk_row_regs<4>(kr, nb, kk, lane, out);
  } else if (nb <= 256) {
    topk_row_regs<8>(kr, nb, kk, lane, out);
  } else if (nb <= 384) {
    topk_row_regs<12>(kr, nb, kk, lane, out);
  } else if (nb <= 512) {
    topk_row_regs<16>(kr, nb, kk, lane, out);
  } else if (nb <= 640) {
    topk_row_regs<20>(kr, nb, kk, lane, out);
  } else if (nb <= 768) {
    topk_row_regs<24>(kr, nb, kk, lane, out);
  } else if (nb <= 896) {
    topk_row_regs<28>(kr, nb, kk, lane, out);
  } else if (nb <= 1024) {
    topk_row_regs<32>(kr, nb, kk, lane, out);
  } else {
    topk_row_smem(kr, nb, kk, lane, out);
  }
}

constexpr int kSelectThreads = 512;  // 16 warps
constexpr int kSelectKT = 128;       // key blocks per score tile

// Shared memory of select_kernel<D> for R query blocks per CTA.
__host__ __device__ constexpr size_t select_smem_bytes(int D, int R, int nb) {
  return ((size_t)32 * D + (size_t)kSelectKT * (D + 4) + 32 + 2 * kSelectKT + (size_t)R * nb) * sizeof(float);
}

// Grid (ceil(nb / R), BH), kSelectThreads threads, R <= 32, dynamic smem:
//   Qb [32][D] fp32 (rows >= R zero), Kc [KT][D+4] fp32, qn [32], mj [KT],
//   nj [KT], keys [R][nb] uint32.
// Phase 1 computes the R x nb scores with fp32 FMAs, KT key blocks at a time;
// each thread holds a 2 x 4 register tile (rows tr, tr+16; key columns
// 64 h + tc + 16c, h the thread's half of the CTA), and stores their orderable
// keys.  The CTA's sixteen warps keep the latency-bound score and selection
// loops busy at one CTA per SM.  Phase 2 runs, per row (one warp per row), an
// MSB-first bitwise search for the k-th largest key, then writes the selected
// indices in ascending order.
template <int D>
__global__ void __launch_bounds__(kSelectThreads)
select_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
              const float* __restrict__ M, int L, int B, int nb, int kk, int R,
              float scale, int32_t* __restrict__ sel) {
  extern __shared__ __align__(16) float sm[];
  constexpr int KS = D + 4;
  constexpr int KT = kSelectKT;                // key blocks per tile
  constexpr int NW = kSelectThreads / 32;      // warps
  float* Qb = sm;                              // 32 * D
  float* Kc = Qb + 32 * D;                     // KT * KS
  float* qn = Kc + KT * KS;                    // 32
  float* mj = qn + 32;                         // KT
  float* nj = mj + KT;                         // KT
  uint32_t* keys = reinterpret_cast<uint32_t*>(nj + KT);  // R * nb
  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * R;
  const int rows = min(R, nb - i0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int e = threadIdx.x; e < 32 * D; e += blockDim.x) {
    const int r = e / D;
    Qb[e] = (r < rows) ? qbar[((size_t)bh * nb + i0 + r) * D + (e % D)] : 0.f;
  }
  __syncthreads();
  for (int r = warp; r < 32; r += NW) {
    float t = 0.f;
    for (int a = lane; a < D; a += 32) t = fmaf(Qb[r * D + a], Qb[r * D + a], t);
    t = warp_sum(t);
    if (lane == 0) qn[r] = sqrtf(t);
  }

  // Phase 1: scores.
  const int tr = (threadIdx.x & 255) >> 4, tc = threadIdx.x & 15, ch = (threadIdx.x >> 8) * 64;
  for (int j0 = 0; j0 < nb; j0 += KT) {
    __syncthreads();
    for (int e = threadIdx.x; e < KT * (D / 4); e += blockDim.x) {
      const int c = e / (D / 4), a = (e % (D / 4)) * 4;
      float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + c < nb) w = *reinterpret_cast<const float4*>(kbar + ((size_t)bh * nb + j0 + c) * D + a);
      *reinterpret_cast<float4*>(Kc + c * KS + a) = w;
    }
    if (threadIdx.x < KT) {
      const int j = j0 + threadIdx.x;
      mj[threadIdx.x] = (j < nb && M != nullptr) ? M[(size_t)bh * nb + j] : 0.f;
      nj[threadIdx.x] = (j < nb) ? (float)min(B, L - j * B) : 1.f;
    }
    __syncthreads();
    float acc[2][4];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
#pragma unroll 4
    for (int a = 0; a < D; a += 4) {
      const float4 q0 = *reinterpret_cast<const float4*>(Qb + tr * D + a);
      const float4 q1 = *reinterpret_cast<const float4*>(Qb + (tr + 16) * D + a);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float4 k = *reinterpret_cast<const float4*>(Kc + (ch + tc + 16 * c) * KS + a);
        acc[0][c] = fmaf(q0.x, k.x, acc[0][c]);
        acc[0][c] = fmaf(q0.y, k.y, acc[0][c]);
        acc[0][c] = fmaf(q0.z, k.z, acc[0][c]);
        acc[0][c] = fmaf(q0.w, k.w, acc[0][c]);
        acc[1][c] = fmaf(q1.x, k.x, acc[1][c]);
        acc[1][c] = fmaf(q1.y, k.y, acc[1][c]);
        acc[1][c] = fmaf(q1.z, k.z, acc[1][c]);
        acc[1][c] = fmaf(q1.w, k.w, acc[1][c]);
      }
    }
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int r = tr + 16 * rr;
      if (r >= rows) continue;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int cl = ch + tc + 16 * c;
        const int j = j0 + cl;
        if (j < nb) keys[r * nb + j] = orderable_key(scale * acc[rr][c] + logf(nj[cl] + scale * qn[r] * mj[cl]));
      }
    }
  }
  __syncthreads();

  // Phase 2: per-row selection, one warp per row.
  for (int r = warp; r < rows; r += NW)
    topk_row_ascending(keys + r * nb, nb, kk, lane, sel + ((size_t)bh * nb + i0 + r) * kk);
}

}  // namespace pisa
