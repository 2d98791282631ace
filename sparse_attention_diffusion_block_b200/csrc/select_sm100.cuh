// Covariance-aware top-k routing with the score GEMM on the 5th-generation
// tensor cores (AI Radio summary of PISA: score Score_{t,j}; gist.science
// technical summary, section 2, covariance-aware routing).  For query block i
// of a (batch, head):
//   score_{i,j} = s qbar_i . kbar_j + ln(n_j + s ||qbar_i||_2 M_j)
//   sel[i]      = the k largest scores, exact ties to the smaller j, ascending.
// With M == nullptr the covariance term drops out (plain pooled routing).
//
// A CTA takes R query blocks of one (batch, head) and all nb key centroids:
//   - the fp32 centroids arrive by TMA in stages of 128 blocks x 64 dims; the
//     split warps read a stage, hand it back to the producer and write it as
//     bf16 hi + lo (x = hi + lo + O(2^-18 |x|)) into tensor memory, where the
//     MMAs read it as their A operand (shared memory carries only the fp32
//     stages and Qbar, no split copy of the centroids);
//   - S^T = Kbar Qbar^T runs as tcgen05 MMAs with M = 128 key blocks, N = R
//     query blocks, as hi.hi + hi.lo + lo.hi: an error of a few 1e-5 in the
//     score for the largest workloads (|s qbar.kbar| ~ 40), well inside the
//     1e-3 score gap the routing inputs keep between the k-th and (k+1)-th
//     block;
//   - each epilogue thread owns one key block (a TMEM lane): it reads the R
//     scores of that block, adds the log term in fp32 and stores orderable
//     keys [R][nb] in shared memory;
//   - then every warp runs the per-row top-k (one warp per query block).
// Warp roles (512 threads): 0-3 epilogue, 4-7 and 12-15 fp32 -> bf16 hi/lo
// split, 8 TMA producer, 9 MMA issuer, all 16 warps for the top-k.
// TMEM columns: [0, 2R) the scores of two key tiles; [128, 256) and [256, 384)
// the hi (first 64 columns) and lo (last 64) centroids of two key tiles.
#pragma once

#include "select.cuh"
#include "sm100.cuh"

namespace pisa {

constexpr int kSelTcThreads = 512;
constexpr uint32_t kSelTcStage = 128u * 64u * 4u;  // 128 key blocks x 64 dims fp32

template <int D, int R>
struct SelectTcLayout {
  static constexpr uint32_t kQ = R * D * 2u;  // Qbar hi (or lo): R rows x D bf16
  __host__ __device__ static size_t keys_bytes(int nb) { return ((size_t)R * nb * 4 + 7) / 8 * 8; }
  static size_t bytes(int ns, int nb) {
    return 1024 + (size_t)ns * kSelTcStage + 2 * kQ + keys_bytes(nb) + R * 4 + (2 * (size_t)ns + 9) * 8 + 16;
  }
};

// x[0..8) -> bf16 hi (RNE) and lo = bf16(x - hi), each as one 16-byte chunk.
__device__ __forceinline__ void split_bf16x8(const float* x, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 hv = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
    const float2 hf = __bfloat1622float2(hv);
    const __nv_bfloat162 lv = __floats2bfloat162_rn(x[2 * e] - hf.x, x[2 * e + 1] - hf.y);
    h[e] = *reinterpret_cast<const uint32_t*>(&hv);
    l[e] = *reinterpret_cast<const uint32_t*>(&lv);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Grid (BH, ceil(nb / R)) when nb is not a multiple of R (heads fastest: the
// CTAs of each head's last, partly filled row tile, with a shorter top-k, run
// last, in the partial wave at the end of the grid), else (ceil(nb / R), BH)
// (a head's CTAs together).  kSelTcThreads threads, dynamic shared memory
// SelectTcLayout<D, R>::bytes(ns, nb); ns >= 2 stages.
// tmK: kbar fp32 [BH][nb][D], boxes of 32 dims x 128 blocks, 128-byte swizzle,
// rows past nb read as zero.
template <int D, int R>
__global__ void __launch_bounds__(kSelTcThreads, 1)
select_sm100_kernel(const __grid_constant__ CUtensorMap tmK, const float* __restrict__ qbar,
                    const float* __restrict__ M, int L, int B, int nb, int kk, int ns, float scale,
                    int32_t* __restrict__ sel) {
  using namespace sm100;
  using Lay = SelectTcLayout<D, R>;
  constexpr int NH = D / 64;                // stages per key tile
  constexpr uint32_t STAGE = kSelTcStage;
  constexpr uint32_t HALF = STAGE / 2;      // the stage's two 32-dim boxes
  constexpr uint32_t QB = R * 128u;         // one 64-dim block of Qbar hi (or lo)
  constexpr uint32_t TCOLS = 512;
  constexpr uint32_t ACOL = 128;            // hi / lo centroid buffers in TMEM
  static_assert(2 * R <= ACOL, "score buffers below the centroid buffers");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sStage = smem;                                   // [ns][STAGE]
  uint8_t* sQh = smem + (size_t)ns * STAGE;                 // [NH][R][128 B]
  uint8_t* sQl = sQh + Lay::kQ;
  uint32_t* keys = reinterpret_cast<uint32_t*>(sQl + Lay::kQ);  // [R][nb]
  float* qn = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(keys) + Lay::keys_bytes(nb));  // [R]
  uint64_t* bars = reinterpret_cast<uint64_t*>(qn + R);
  uint64_t* full = bars;              // [ns] fp32 stage landed
  uint64_t* empty = bars + ns;        // [ns] stage read by the split warps
  uint64_t* a_full = bars + 2 * ns;   // [2] hi / lo centroids of a key tile in TMEM
  uint64_t* a_empty = a_full + 2;     // [2] ... read by the MMAs
  uint64_t* d_full = a_empty + 2;     // [2] scores of a key tile in TMEM
  uint64_t* d_empty = d_full + 2;     // [2] scores read out of TMEM
  uint64_t* mma_idle = d_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_idle + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const bool heads_fast = (nb % R) != 0;
  const int bh = heads_fast ? blockIdx.x : blockIdx.y;
  const int i0 = (heads_fast ? blockIdx.y : blockIdx.x) * R;
  const int rows = min(R, nb - i0);
  const int ntiles = (nb + 127) / 128;
  const int nit = ntiles * NH;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ns; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);  // the four split warps of the stage's half
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&a_full[x], 4 * NH);
      mbar_init(&a_empty[x], 1);
      mbar_init(&d_full[x], 1);
      mbar_init(&d_empty[x], 128);
    }
    mbar_init(mma_idle, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, TCOLS);
    tmem_relinquish();
  }
  // Qbar rows of this CTA as bf16 hi / lo, K-major with the 128-byte swizzle
  // (16-byte chunk c of row r at position c ^ (r mod 8)); rows past nb are
  // zero.  The D/8 threads of a row (consecutive lanes) also sum its squares.
  static_assert(R * (D / 8) <= kSelTcThreads, "one 8-dim chunk per thread");
  {
    const int c = threadIdx.x;
    const int r = c / (D / 8), c8 = c % (D / 8);
    float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (c < R * (D / 8) && r < rows) load8(qbar + ((size_t)bh * nb + i0 + r) * D + 8 * c8, x);
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
    for (int o = 1; o < D / 8; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (c < R * (D / 8)) {
      uint4 hi, lo;
      split_bf16x8(x, hi, lo);
      const uint32_t off = (c8 / 8) * QB + r * 128u + (((c8 % 8) ^ (r & 7)) << 4);
      *reinterpret_cast<uint4*>(sQh + off) = hi;
      *reinterpret_cast<uint4*>(sQl + off) = lo;
      if (c8 == 0) qn[r] = sqrtf(ss);
    }
  }
  fence_proxy_async_smem();
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ================================================================ producer
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      int it = 0;
      for (; it < nit; ++it) {
        const int s = it % ns;
        if (!mbar_wait(&empty[s], ((it / ns) & 1) ^ 1, abort)) break;
        const int t = it / NH, h = it % NH;
        mbar_expect_tx(&full[s], STAGE);
        tma_load_3d(sStage + s * STAGE, &tmK, &full[s], h * 64, t * 128, bh);
        tma_load_3d(sStage + s * STAGE + HALF, &tmK, &full[s], h * 64 + 32, t * 128, bh);
      }
      // the last load of each stage lands before the CTA can exit
      for (int u = it > ns ? it - ns : 0; u < it; ++u) mbar_drain(&full[u % ns], (u / ns) & 1);
    }
  } else if ((warp >= 4 && warp < 8) || warp >= 12) {
    // ================================================================ hi / lo split into TMEM
    // Warp w owns TMEM lane quarter q = w % 4, i.e. key blocks 32 q + lane of
    // each tile, and the stages of dim half c (warps 4-7: dims 0-63, warps
    // 12-15: dims 64-127).  Lane l reads its row's 64 fp32 from the stage,
    // the warp hands the stage back to the producer, and the row goes to
    // TMEM as 32 columns of bf16x2 hi and 32 of lo (dims 2w, 2w+1 in column
    // w of the half).
    const int q = warp % 4, c = warp < 8 ? 0 : 1;
    const int r = 32 * q + lane;
    const uint32_t rsw = r & 7;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    for (int it = c; c < NH && it < nit; it += NH) {
      const int s = it % ns, t = it / NH, buf = t & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (it / ns) & 1, abort))) break;
      const uint8_t* st = sStage + s * STAGE;
      float4 v[16];  // v[8 b + k]: chunk k of box b (dims 32 b + 4 k ..)
#pragma unroll
      for (int k = 0; k < 16; ++k)
        v[k] = *reinterpret_cast<const float4*>(st + (k / 8) * HALF + r * 128u + (((k % 8) ^ rsw) << 4));
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      // the MMAs of tile t - 2 have read this TMEM buffer
      if (t >= 2 && !__all_sync(0xffffffffu, mbar_wait(&a_empty[buf], ((t >> 1) - 1) & 1, abort))) break;
      const uint32_t ab = tmem + lane_off + ACOL + buf * 128 + c * 32;
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        uint32_t hw[16], lw[16];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float4 x0 = v[8 * b + 2 * g], x1 = v[8 * b + 2 * g + 1];
          const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          uint4 hi, lo;
          split_bf16x8(x, hi, lo);
          hw[4 * g] = hi.x, hw[4 * g + 1] = hi.y, hw[4 * g + 2] = hi.z, hw[4 * g + 3] = hi.w;
          lw[4 * g] = lo.x, lw[4 * g + 1] = lo.y, lw[4 * g + 2] = lo.z, lw[4 * g + 3] = lo.w;
        }
        tmem_st16(ab + 16 * b, hw);
        tmem_st16(ab + 64 + 16 * b, lw);
      }
      tmem_wait_st();
      fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[buf]);
    }
  } else if (warp == 9) {
    // ================================================================ MMA issuer
    // A (centroid hi / lo) from TMEM, B (Qbar hi / lo) from shared memory; the
    // three products of each 16-dim step in the same order as always.
    constexpr uint32_t idS = idesc_bf16(128, R, false, false);
    const uint32_t qh = smem_u32(sQh), ql = smem_u32(sQl);
    bool ok = true;
    for (int t = 0; ok && t < ntiles; ++t) {
      const int buf = t & 1;
      if (!(ok = mbar_wait(&a_full[buf], (t >> 1) & 1, abort))) break;
      if (t >= 2 && !(ok = mbar_wait(&d_empty[buf], ((t >> 1) - 1) & 1, abort))) break;
      fence_after_sync();
      const uint32_t d = tmem + buf * R;
      const uint32_t ah = tmem + ACOL + buf * 128, al = ah + 64;
      for (int h = 0; h < NH; ++h) {
        const uint32_t bhq = qh + h * QB, blq = ql + h * QB;
#pragma unroll
        for (int kk16 = 0; kk16 < 4; ++kk16) {
          const uint32_t ac = (h * 4 + kk16) * 8;
          const uint64_t bdh = desc_sw128(bhq + kk16 * 32, 16, 1024), bdl = desc_sw128(blq + kk16 * 32, 16, 1024);
          mma_ts_warp(d, ah + ac, bdh, idS, (h > 0 || kk16 > 0) ? 1u : 0u);
          mma_ts_warp(d, ah + ac, bdl, idS, 1u);
          mma_ts_warp(d, al + ac, bdh, idS, 1u);
        }
      }
      mma_commit_warp(&d_full[buf]);
      mma_commit_warp(&a_empty[buf]);
    }
    mma_commit_warp(mma_idle);
    mbar_drain(mma_idle, 0);
    __syncwarp();
  } else if (warp < 4) {
    // ================================================================ epilogue
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float sq[R];  // s ||qbar_r||, in registers for the whole loop
#pragma unroll
    for (int r = 0; r < R; ++r) sq[r] = scale * qn[r];
    for (int t = 0; t < ntiles; ++t) {
      const int buf = t & 1;
      const int j = t * 128 + threadIdx.x;
      // this key block's size and covariance norm, loaded before the wait
      const float nj = j < nb ? (float)min(B, L - j * B) : 1.f;
      const float mj = (M != nullptr && j < nb) ? M[(size_t)bh * nb + j] : 0.f;
      if (!__all_sync(0xffffffffu, mbar_wait(&d_full[buf], (t >> 1) & 1, abort))) break;
      fence_after_sync();
      uint32_t acc[R];
      if constexpr (R == 32) {
        tmem_ld32(lane_base + buf * R, acc);
      } else {
        tmem_ld16(lane_base + buf * R, acc);
      }
      tmem_wait_ld();
      fence_before_sync();
      mbar_arrive(&d_empty[buf]);
      if (j < nb) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          if (r < rows)
            keys[r * nb + j] =
                orderable_key(fmaf(scale, __uint_as_float(acc[r]), __logf(fmaf(sq[r], mj, nj))));
        }
      }
    }
  }

  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (!*abort) {
    // per-row selection, one warp per query block
    for (int r = warp; r < rows; r += kSelTcThreads / 32)
      topk_row_ascending(keys + r * nb, nb, kk, lane, sel + ((size_t)bh * nb + i0 + r) * kk);
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 9) tmem_dealloc(tmem, TCOLS);
}

}  // namespace pisa
