// Fused PISA forward on CUDA cores (fp32 inputs).
//
// gist.science technical summary of PISA, section 2: core algorithm (the N_t
// equation with alpha_{t,j} = exp(q_t kbar_j^T)) and hardware implementation
// (phase 1 exact attention over the selected blocks, phase 2 zeroth-order
// scan of the unselected blocks' aggregated vectors, phase 3 the global
// first-order correction), all inside one online softmax: a single running
// max m_t, denominator l_t = D_t e^{-m_t}, numerator O_t = N_t e^{-m_t} and
// beta_t e^{-m_t}; the approximation never forms a separate branch.
#pragma once

#include "common.cuh"

namespace pisa {

// o[0..DS) += fo * (q_t H)[sl*DS .. sl*DS+DS) for the row whose TPR threads
// hold q_t in slices: each thread forms the partial products of its own slice
// of q_t with every column block, and the TPR partials of a column block are
// summed with shuffles.  Hs: a D x D matrix in shared memory (row = key dim).
template <int D, int TPR>
__device__ __forceinline__ void add_q_times_h(const float* __restrict__ Hs, const float* qr, float* o, float fo,
                                              int sl) {
  constexpr int DS = D / TPR;
#pragma unroll 1
  for (int g = 0; g < TPR; ++g) {
    float part[DS];
#pragma unroll
    for (int c = 0; c < DS; ++c) part[c] = 0.f;
#pragma unroll 4
    for (int a = 0; a < DS; ++a) {
      const float qa = qr[a];
      const float* hrow = Hs + (sl * DS + a) * D + g * DS;
#pragma unroll
      for (int c = 0; c < DS; c += 4) {
        const float4 w = *reinterpret_cast<const float4*>(hrow + c);
        part[c] = fmaf(qa, w.x, part[c]);
        part[c + 1] = fmaf(qa, w.y, part[c + 1]);
        part[c + 2] = fmaf(qa, w.z, part[c + 2]);
        part[c + 3] = fmaf(qa, w.w, part[c + 3]);
      }
    }
#pragma unroll
    for (int c = 0; c < DS; ++c) {
#pragma unroll
      for (int off = 1; off < TPR; off <<= 1) part[c] += __shfl_xor_sync(0xffffffffu, part[c], off);
    }
    if (sl == g) {
#pragma unroll
      for (int c = 0; c < DS; ++c) o[c] = fmaf(fo, part[c], o[c]);
    }
  }
}

// One CTA per (query block i, bh); TPR threads per query row, each owning
// DS = D / TPR consecutive dimensions of q_t and O_t.  Keys are staged in
// shared memory CH at a time, fp32, laid out [CH][TPR][DS + 4].
//
// BLOCKWISE selects the first-order term before hybridisation (gist.science
// summary, section 2, the hybrid-order paragraph starts from it): every
// unselected block keeps its own H_j, N_t += s alpha_{t,j} (q_t H_j), instead
// of the shared s beta_t (q_t Hbar).  `first` is then H [BH][nb][D][D]; the
// term is folded into the same running numerator as the block's value sum.
// It costs |U_i| D^2 multiply-adds per row: a comparison variant for small
// shapes, not the production path.  Otherwise `first` is Hbar [BH][D][D].
template <typename T, int D, int TPR, int CH, bool BLOCKWISE = false>
__global__ void __launch_bounds__(512, 1)
fused_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  T* __restrict__ out, int L, int B, int nb, int kk,
                  const float* __restrict__ kbar, const float* __restrict__ vsum,
                  const float* __restrict__ first, const int32_t* __restrict__ sel, float scale) {
  constexpr int DS = D / TPR;
  constexpr int SS = DS + 4;            // padded slice stride
  constexpr int RS = TPR * SS;          // padded row stride
  extern __shared__ __align__(16) float sm[];
  float* Kt = sm;                       // CH * RS
  float* Vt = Kt + CH * RS;             // CH * RS
  float* Hs = Vt + CH * RS;             // D * D   (Hbar)
  float* nj_s = Hs + D * D;             // CH
  uint32_t* mask = reinterpret_cast<uint32_t*>(nj_s + CH);  // ceil(nb/32) words: S_i membership

  const int i = blockIdx.x, bh = blockIdx.y;
  const int r = threadIdx.x / TPR, sl = threadIdx.x % TPR;
  const int row0 = i * B, n_i = min(B, L - row0);
  const bool active = r < n_i;
  const size_t base = (size_t)bh * L * D;
  const float c2 = scale * kLog2e;      // exponents in base 2
  const int words = (nb + 31) / 32;

  for (int w = threadIdx.x; w < words; w += blockDim.x) mask[w] = 0u;
  __syncthreads();
  const int32_t* si = sel + ((size_t)bh * nb + i) * kk;
  for (int e = threadIdx.x; e < kk; e += blockDim.x) {
    const int j = si[e];
    if (j < 0 || j >= nb) {
      raise_device_error(PISA_ERR_DEVICE_CHECK);
    } else {
      atomicOr(&mask[j >> 5], 1u << (j & 31));
    }
  }

  float qr[DS], o[DS];
#pragma unroll
  for (int e = 0; e < DS; e += 8) {
    if (active) {
      load8(q + base + (size_t)(row0 + r) * D + sl * DS + e, qr + e);
    } else {
#pragma unroll
      for (int x = 0; x < 8; ++x) qr[e + x] = 0.f;
    }
  }
#pragma unroll
  for (int e = 0; e < DS; ++e) o[e] = 0.f;
  float m = -INFINITY, l = 0.f, beta = 0.f;

  // ---- phase 1: exact attention over the selected blocks
  for (int e = 0; e < kk; ++e) {
    const int j = si[e];
    if (j < 0 || j >= nb) continue;
    const int n_j = min(B, L - j * B);
    for (int c0 = 0; c0 < n_j; c0 += CH) {
      const int cn = min(CH, n_j - c0);
      __syncthreads();
      for (int g = threadIdx.x; g < CH * (D / 8); g += blockDim.x) {
        const int rr = g / (D / 8), cc = (g % (D / 8)) * 8;
        float xk[8], xv[8];
        if (rr < cn) {
          const size_t off = base + (size_t)(j * B + c0 + rr) * D + cc;
          load8(k + off, xk);
          load8(v + off, xv);
        } else {
#pragma unroll
          for (int x = 0; x < 8; ++x) xk[x] = xv[x] = 0.f;
        }
        const int so = rr * RS + (cc / DS) * SS + (cc % DS);
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          Kt[so + x] = xk[x];
          Vt[so + x] = xv[x];
        }
      }
      __syncthreads();
      float x[CH];
      float cmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        float part = 0.f;
        const float* kr = Kt + c * RS + sl * SS;
#pragma unroll
        for (int e2 = 0; e2 < DS; e2 += 4) {
          const float4 y = *reinterpret_cast<const float4*>(kr + e2);
          part = fmaf(qr[e2], y.x, part);
          part = fmaf(qr[e2 + 1], y.y, part);
          part = fmaf(qr[e2 + 2], y.z, part);
          part = fmaf(qr[e2 + 3], y.w, part);
        }
#pragma unroll
        for (int off = 1; off < TPR; off <<= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        x[c] = (c < cn) ? part * c2 : -INFINITY;
        cmax = fmaxf(cmax, x[c]);
      }
      const float m_new = fmaxf(m, cmax);
      const float corr = exp2f(m - m_new);
      l *= corr;
#pragma unroll
      for (int e2 = 0; e2 < DS; ++e2) o[e2] *= corr;
      m = m_new;
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const float p = exp2f(x[c] - m);
        l += p;
        const float* vr = Vt + c * RS + sl * SS;
#pragma unroll
        for (int e2 = 0; e2 < DS; e2 += 4) {
          const float4 y = *reinterpret_cast<const float4*>(vr + e2);
          o[e2] = fmaf(p, y.x, o[e2]);
          o[e2 + 1] = fmaf(p, y.y, o[e2 + 1]);
          o[e2 + 2] = fmaf(p, y.z, o[e2 + 2]);
          o[e2 + 3] = fmaf(p, y.w, o[e2 + 3]);
        }
      }
    }
  }

  // ---- phase 2: zeroth-order terms of the unselected blocks
  const float* kb = kbar + (size_t)bh * nb * D;
  const float* vs = vsum + (size_t)bh * nb * D;
  for (int j0 = 0; j0 < nb; j0 += CH) {
    const int cn = min(CH, nb - j0);
    __syncthreads();
    for (int g = threadIdx.x; g < CH * D; g += blockDim.x) {
      const int rr = g / D, cc = g % D;
      const int so = rr * RS + (cc / DS) * SS + (cc % DS);
      Kt[so] = (rr < cn) ? kb[(size_t)(j0 + rr) * D + cc] : 0.f;
      Vt[so] = (rr < cn) ? vs[(size_t)(j0 + rr) * D + cc] : 0.f;
    }
    if (threadIdx.x < CH) {
      const int j = j0 + threadIdx.x;
      nj_s[threadIdx.x] = (j < nb) ? (float)min(B, L - j * B) : 0.f;
    }
    __syncthreads();
    float y[CH];
    float cmax = -INFINITY;
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      float part = 0.f;
      const float* kr = Kt + c * RS + sl * SS;
#pragma unroll
      for (int e2 = 0; e2 < DS; e2 += 4) {
        const float4 w = *reinterpret_cast<const float4*>(kr + e2);
        part = fmaf(qr[e2], w.x, part);
        part = fmaf(qr[e2 + 1], w.y, part);
        part = fmaf(qr[e2 + 2], w.z, part);
        part = fmaf(qr[e2 + 3], w.w, part);
      }
#pragma unroll
      for (int off = 1; off < TPR; off <<= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      const int j = j0 + c;
      const bool use = (c < cn) && !((mask[j >> 5] >> (j & 31)) & 1u);
      y[c] = use ? part * c2 : -INFINITY;
      cmax = fmaxf(cmax, y[c]);
    }
    const float m_new = fmaxf(m, cmax);
    // nothing unselected in this tile yet (uniform: the CTA's rows share S_i)
    if (m_new == -INFINITY && !BLOCKWISE) continue;
    const float corr = m_new == -INFINITY ? 1.f : exp2f(m - m_new);
    l *= corr;
    beta *= corr;
#pragma unroll
    for (int e2 = 0; e2 < DS; ++e2) o[e2] *= corr;
    m = m_new;
    float alpha[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
      const float a = m == -INFINITY ? 0.f : exp2f(y[c] - m);
      alpha[c] = a;
      beta += a;
      l = fmaf(nj_s[c], a, l);
      const float* vr = Vt + c * RS + sl * SS;
#pragma unroll
      for (int e2 = 0; e2 < DS; e2 += 4) {
        const float4 w = *reinterpret_cast<const float4*>(vr + e2);
        o[e2] = fmaf(a, w.x, o[e2]);
        o[e2 + 1] = fmaf(a, w.y, o[e2 + 1]);
        o[e2 + 2] = fmaf(a, w.z, o[e2 + 2]);
        o[e2 + 3] = fmaf(a, w.w, o[e2 + 3]);
      }
    }
    if constexpr (BLOCKWISE) {
      // each unselected block's own first-order term, weighted like its value
      // sum: O += s alpha_{t,j} (q_t H_j)
      for (int c = 0; c < cn; ++c) {
        const int j = j0 + c;
        if ((mask[j >> 5] >> (j & 31)) & 1u) continue;  // selected: exact above
        __syncthreads();
        const float* hj = first + ((size_t)bh * nb + j) * D * D;
        for (int e = threadIdx.x; e < D * D / 4; e += blockDim.x)
          reinterpret_cast<float4*>(Hs)[e] = reinterpret_cast<const float4*>(hj)[e];
        __syncthreads();
        add_q_times_h<D, TPR>(Hs, qr, o, scale * alpha[c], sl);
      }
    }
  }

  if constexpr (!BLOCKWISE) {
    // ---- phase 3: global first-order correction  O += s * beta * (q Hbar)
    __syncthreads();
    const float* hb = first + (size_t)bh * D * D;
    for (int e = threadIdx.x; e < D * D; e += blockDim.x) Hs[e] = hb[e];
    __syncthreads();
    add_q_times_h<D, TPR>(Hs, qr, o, scale * beta, sl);
  }

  if (active) {
    const float inv = 1.f / l;
    T* dst = out + base + (size_t)(row0 + r) * D + sl * DS;
#pragma unroll
    for (int e = 0; e < DS; ++e) dst[e] = from_float<T>(o[e] * inv);
  }
}

}  // namespace pisa
