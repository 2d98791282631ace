// Block statistics and covariance norms on the tensor cores (bf16 inputs, d = 128).
//
// gist.science technical summary of PISA, section 2: hardware implementation
// ("precompute" of block centroids, value sums and the global statistic Hbar)
// and covariance-aware routing (M_j = ||H_j - Hbar||).
//
// Both kernels stream Q/K/V tiles with TMA and run the contractions over the
// tokens of a block as tcgen05 MMAs with MN-major operands:
//   column sums    X_j^T 1   (M = d, N = 16, K = block tokens)  -> qbar, kbar, vsum
//   first order    K_j^T V_j (M = d, N = d,  K = block tokens)
// bf16 products are exact in the fp32 accumulator, so H_j = K_j^T V_j -
// kbar_j^T vsum_j is formed without rounding centred keys to bf16.
#pragma once

#include "sm100.cuh"

namespace pisa {

constexpr int kStatsThreads = 192;
constexpr int kStatsStages = 6;

template <int KB>
struct StatsLayout {
  static constexpr int D = 128;
  static constexpr uint32_t kTile = KB * D * 2u;        // one Q/K/V tile of a block
  static constexpr uint32_t kRing = kStatsStages * kTile;
  static constexpr uint32_t kOnes = 16 * KB * 2u;        // 16 x KB ones (K-major)
  static constexpr uint32_t kSig = 3 * D * 4u;           // value-sum exchange (2 buffers in the stats kernel, 3 in cov)
  static constexpr uint32_t kRed = 2 * 8 * 4u;           // cross-warp partials, double buffered
  static constexpr uint32_t kBars = (2 * kStatsStages + 13) * 8u;
  static constexpr size_t bytes() { return 1024 + kRing + kOnes + kSig + kRed + kBars + 16; }
};

// Descriptor of an MN-major operand held as [rows][128] bf16 in two 64-column
// swizzled blocks, rows = contraction dimension; k-step kk covers rows 16kk..16kk+15.
__device__ __forceinline__ uint64_t desc_mn(uint32_t base, int rows, int kk) {
  return sm100::desc_sw128(base + kk * 16 * 128, rows * 128, 1024);
}

// Grid (n_chunks, BH).  A CTA walks J consecutive blocks of one (batch, head):
// writes qbar/kbar/vsum of each block and its chunk partial
//   sum_j (K_j^T V_j - kbar_j^T vsum_j)   [d x d], fixed order.
template <int KB>
__global__ void __launch_bounds__(kStatsThreads, 1)
stats_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, int L, int nb, int J, float* __restrict__ qbar,
                   float* __restrict__ kbar, float* __restrict__ vsum, float* __restrict__ partial) {
  using namespace sm100;
  using Lay = StatsLayout<KB>;
  constexpr int D = 128, NS = kStatsStages;
  constexpr uint32_t TILE = Lay::kTile;
  constexpr uint32_t HC = 0, SUMC = 128;  // TMEM: H [0,128), sums [128, 224)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sRing = smem;
  uint8_t* sOnes = smem + Lay::kRing;
  float* sig = reinterpret_cast<float*>(sOnes + Lay::kOnes);  // [2][D]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sig) + Lay::kSig + Lay::kRed);
  uint64_t* full = bars;
  uint64_t* empty = bars + NS;
  uint64_t* sums_full = bars + 2 * NS;  // [2]
  uint64_t* sums_free = sums_full + 2;  // [2]
  uint64_t* h_final = sums_free + 2;
  uint64_t* mma_idle = h_final + 1;
  uint64_t* sig_full = mma_idle + 1;  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 10);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int j0 = chunk * J;
  const int nj = min(J, nb - j0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&sums_full[0], 1);
    mbar_init(&sums_full[1], 1);
    mbar_init(&sums_free[0], 128);
    mbar_init(&sums_free[1], 128);
    mbar_init(&sig_full[0], 128);
    mbar_init(&sig_full[1], 128);
    mbar_init(h_final, 1);
    mbar_init(mma_idle, 1);
    *abort = 0;
    fence_mbar_init();
  }
  {
    // ones operand (any layout of ones is the same matrix)
    uint32_t* o = reinterpret_cast<uint32_t*>(sOnes);
    for (int e = threadIdx.x; e < (int)(Lay::kOnes / 4); e += blockDim.x) o[e] = 0x3F803F80u;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      int it = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* map, int row) -> bool {
        const int s = it % NS;
        if (!mbar_wait(&empty[s], ((it / NS) & 1) ^ 1, abort)) return false;
        mbar_expect_tx(&full[s], TILE);
        tma_load_3d(sRing + s * TILE, map, &full[s], 0, row, bh);
        tma_load_3d(sRing + s * TILE + KB * 128, map, &full[s], 64, row, bh);
        ++it;
        return true;
      };
      for (int jj = 0; ok && jj < nj; ++jj) {
        const int row = (j0 + jj) * KB;
        ok = load(&tmQ, row) && load(&tmK, row) && load(&tmV, row);
      }
      {
        // the last load of each ring slot lands before the CTA can exit (after
        // another role gave up nothing else waits for it)
        const int first = it > NS ? it - NS : 0;
        for (int u = first; u < it; ++u) mbar_drain(&full[u % NS], (u / NS) & 1);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t idSum = idesc_bf16(128, 16, true, false);
      constexpr uint32_t idH = idesc_bf16(128, 128, true, true);
      const uint32_t ring = smem_u32(sRing);
      const uint32_t ones = smem_u32(sOnes);
      auto ones_desc = [&](int kk) { return desc_sw128(ones + (kk >> 2) * 16 * 128 + (kk & 3) * 32, 16, 1024); };
      int it = 0;
      auto take = [&](int& s) -> bool {
        s = it % NS;
        if (!mbar_wait(&full[s], (it / NS) & 1, abort)) return false;
        fence_after_sync();
        ++it;
        return true;
      };
      bool ok = true;
      for (int jj = 0; ok && jj < nj; ++jj) {
        const int buf = jj & 1;
        if (jj >= 2) {
          ok = mbar_wait(&sums_free[buf], ((jj >> 1) - 1) & 1, abort);
          if (!ok) break;
          fence_after_sync();
        }
        const uint32_t sc = tmem + SUMC + buf * 48;
        int sq, sk, sv;
        if (!(ok = take(sq))) break;
        for (int kk = 0; kk < KB / 16; ++kk)
          mma_ss(sc, desc_mn(ring + sq * TILE, KB, kk), ones_desc(kk), idSum, kk > 0 ? 1u : 0u);
        mma_commit(&empty[sq]);
        if (!(ok = take(sk))) break;
        for (int kk = 0; kk < KB / 16; ++kk)
          mma_ss(sc + 16, desc_mn(ring + sk * TILE, KB, kk), ones_desc(kk), idSum, kk > 0 ? 1u : 0u);
        if (!(ok = take(sv))) break;
        for (int kk = 0; kk < KB / 16; ++kk)
          mma_ss(sc + 32, desc_mn(ring + sv * TILE, KB, kk), ones_desc(kk), idSum, kk > 0 ? 1u : 0u);
        for (int kk = 0; kk < KB / 16; ++kk)
          mma_ss(tmem + HC, desc_mn(ring + sk * TILE, KB, kk), desc_mn(ring + sv * TILE, KB, kk), idH,
                 (jj > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[sk]);
        mma_commit(&empty[sv]);
        mma_commit(&sums_full[buf]);
      }
      if (ok) mma_commit(h_final);
      mma_commit(mma_idle);
      mbar_drain(mma_idle, 0);
    }
    __syncwarp();
  } else {
    // warps 0-3: thread a owns dimension a (TMEM lane a)
    const int a = threadIdx.x;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float acc[D];
#pragma unroll
    for (int b = 0; b < D; ++b) acc[b] = 0.f;
    bool ok = true;
    for (int jj = 0; jj < nj; ++jj) {
      const int buf = jj & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&sums_full[buf], (jj >> 1) & 1, abort))) {
        ok = false;
        break;
      }
      fence_after_sync();
      const uint32_t sc = lane_base + SUMC + buf * 48;
      const float sq = __uint_as_float(tmem_ld1(sc));
      const float sk = __uint_as_float(tmem_ld1(sc + 16));
      const float sv = __uint_as_float(tmem_ld1(sc + 32));
      tmem_wait_ld();
      const int j = j0 + jj;
      const float n = (float)min(KB, L - j * KB);
      const size_t o = ((size_t)bh * nb + j) * D + a;
      const float kb = sk / n;
      qbar[o] = sq / n;
      kbar[o] = kb;
      vsum[o] = sv;
      // every thread needs the whole vsum_j: exchange through smem.  The buffer
      // is rewritten two blocks later, only after all 128 threads have arrived
      // on sums_free below (the MMA for that block waits for it).
      sig[buf * D + a] = sv;
      mbar_arrive(&sig_full[buf]);
      if (!__all_sync(0xffffffffu, mbar_wait(&sig_full[buf], (jj >> 1) & 1, abort))) {
        ok = false;
        break;
      }
      const float4* s4 = reinterpret_cast<const float4*>(sig + buf * D);
#pragma unroll
      for (int b = 0; b < D / 4; ++b) {
        const float4 w = s4[b];
        acc[4 * b] = fmaf(kb, w.x, acc[4 * b]);
        acc[4 * b + 1] = fmaf(kb, w.y, acc[4 * b + 1]);
        acc[4 * b + 2] = fmaf(kb, w.z, acc[4 * b + 2]);
        acc[4 * b + 3] = fmaf(kb, w.w, acc[4 * b + 3]);
      }
      fence_before_sync();
      mbar_arrive(&sums_free[buf]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(h_final, 0, abort))) {
      fence_after_sync();
      float* dst = partial + (((size_t)bh * gridDim.x + chunk) * D + a) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t h[32];
        tmem_ld32(lane_base + HC + ch * 32, h);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + ch * 32 + e) =
              make_float4(__uint_as_float(h[e]) - acc[ch * 32 + e], __uint_as_float(h[e + 1]) - acc[ch * 32 + e + 1],
                          __uint_as_float(h[e + 2]) - acc[ch * 32 + e + 2],
                          __uint_as_float(h[e + 3]) - acc[ch * 32 + e + 3]);
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 5) tmem_dealloc(tmem, 256);
}

// Grid (n_chunks, BH).  For each of J consecutive blocks: H_j = K_j^T V_j -
// kbar_j^T vsum_j recomputed on the tensor cores (double-buffered in TMEM),
// M_j = ||H_j - Hbar||_F reduced over the 128 epilogue threads in fixed order.
template <int KB>
__global__ void __launch_bounds__(kStatsThreads, 1)
cov_norm_sm100_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, int L,
                      int nb, int J, const float* __restrict__ kbar, const float* __restrict__ vsum,
                      const float* __restrict__ hbar, float* __restrict__ M) {
  using namespace sm100;
  using Lay = StatsLayout<KB>;
  constexpr int D = 128, NS = kStatsStages;
  constexpr uint32_t TILE = Lay::kTile;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sRing = smem;
  float* sig = reinterpret_cast<float*>(smem + Lay::kRing + Lay::kOnes);  // [2][D]
  float* red = sig + Lay::kSig / 4;  // [2][8]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sig) + Lay::kSig + Lay::kRed);
  uint64_t* full = bars;
  uint64_t* empty = bars + NS;
  uint64_t* d_full = bars + 2 * NS;  // [2]
  uint64_t* d_free = d_full + 2;     // [2]
  uint64_t* mma_idle = d_free + 2;
  uint64_t* red_full = mma_idle + 1;  // [2]
  uint64_t* vs_full = red_full + 2;   // [3] value sum of a block staged in sig
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 13);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int j0 = chunk * J;
  const int nj = min(J, nb - j0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int x = 0; x < 3; ++x) mbar_init(&vs_full[x], 128);
    mbar_init(&d_full[0], 1);
    mbar_init(&d_full[1], 1);
    mbar_init(&d_free[0], 128);
    mbar_init(&d_free[1], 128);
    mbar_init(&red_full[0], 4);
    mbar_init(&red_full[1], 4);
    mbar_init(mma_idle, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      int it = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* map, int row) -> bool {
        const int s = it % NS;
        if (!mbar_wait(&empty[s], ((it / NS) & 1) ^ 1, abort)) return false;
        mbar_expect_tx(&full[s], TILE);
        tma_load_3d(sRing + s * TILE, map, &full[s], 0, row, bh);
        tma_load_3d(sRing + s * TILE + KB * 128, map, &full[s], 64, row, bh);
        ++it;
        return true;
      };
      for (int jj = 0; ok && jj < nj; ++jj) {
        const int row = (j0 + jj) * KB;
        ok = load(&tmK, row) && load(&tmV, row);
      }
      {
        // the last load of each ring slot lands before the CTA can exit (after
        // another role gave up nothing else waits for it)
        const int first = it > NS ? it - NS : 0;
        for (int u = first; u < it; ++u) mbar_drain(&full[u % NS], (u / NS) & 1);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t idH = idesc_bf16(128, 128, true, true);
      const uint32_t ring = smem_u32(sRing);
      int it = 0;
      auto take = [&](int& s) -> bool {
        s = it % NS;
        if (!mbar_wait(&full[s], (it / NS) & 1, abort)) return false;
        fence_after_sync();
        ++it;
        return true;
      };
      bool ok = true;
      for (int jj = 0; ok && jj < nj; ++jj) {
        const int buf = jj & 1;
        if (jj >= 2) {
          ok = mbar_wait(&d_free[buf], ((jj >> 1) - 1) & 1, abort);
          if (!ok) break;
          fence_after_sync();
        }
        int sk, sv;
        if (!(ok = take(sk) && take(sv))) break;
        for (int kk = 0; kk < KB / 16; ++kk)
          mma_ss(tmem + buf * 128, desc_mn(ring + sk * TILE, KB, kk), desc_mn(ring + sv * TILE, KB, kk), idH,
                 kk > 0 ? 1u : 0u);
        mma_commit(&empty[sk]);
        mma_commit(&empty[sv]);
        mma_commit(&d_full[buf]);
      }
      mma_commit(mma_idle);
      mbar_drain(mma_idle, 0);
    }
    __syncwarp();
  } else {
    const int a = threadIdx.x;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float hb[D];
    const float* hrow = hbar + ((size_t)bh * D + a) * D;
#pragma unroll
    for (int b = 0; b < D; b += 4) {
      const float4 w = *reinterpret_cast<const float4*>(hrow + b);
      hb[b] = w.x;
      hb[b + 1] = w.y;
      hb[b + 2] = w.z;
      hb[b + 3] = w.w;
    }
    // this thread's kbar and vsum entries of the next block, loaded one block
    // ahead so their latency hides behind the current block's epilogue
    const size_t ob = ((size_t)bh * nb + j0) * D + a;
    float kb_next = kbar[ob], vs_next = vsum[ob];
    for (int jj = 0; jj < nj; ++jj) {
      const int buf = jj & 1;
      const int j = j0 + jj;
      const float kb = kb_next, vs = vs_next;
      if (jj + 1 < nj) {
        kb_next = kbar[ob + (size_t)(jj + 1) * D];
        vs_next = vsum[ob + (size_t)(jj + 1) * D];
      }
      // every thread needs the whole vsum_j: staged in shared memory before
      // the wait for H_j.  Three buffers: a thread starting block jj knows
      // every epilogue thread has finished block jj - 3 (the MMA of jj - 1
      // waited for d_free of jj - 3).
      const int vb = jj % 3;
      sig[vb * D + a] = vs;
      mbar_arrive(&vs_full[vb]);
      const float4* s4 = reinterpret_cast<const float4*>(sig + vb * D);
      if (!__all_sync(0xffffffffu, mbar_wait(&d_full[buf], (jj >> 1) & 1, abort))) break;
      if (!__all_sync(0xffffffffu, mbar_wait(&vs_full[vb], (jj / 3) & 1, abort))) break;
      fence_after_sync();
      // four independent partial sums (columns b mod 4), added in a fixed order
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t h[32];
        tmem_ld32(lane_base + buf * 128 + ch * 32, h);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 w = s4[(ch * 32 + e) / 4];
          const float d0 = __uint_as_float(h[e]) - fmaf(kb, w.x, hb[ch * 32 + e]);
          const float d1 = __uint_as_float(h[e + 1]) - fmaf(kb, w.y, hb[ch * 32 + e + 1]);
          const float d2 = __uint_as_float(h[e + 2]) - fmaf(kb, w.z, hb[ch * 32 + e + 2]);
          const float d3 = __uint_as_float(h[e + 3]) - fmaf(kb, w.w, hb[ch * 32 + e + 3]);
          s0 = fmaf(d0, d0, s0);
          s1 = fmaf(d1, d1, s1);
          s2 = fmaf(d2, d2, s2);
          s3 = fmaf(d3, d3, s3);
        }
      }
      float ss = (s0 + s1) + (s2 + s3);
      // fixed-order reduction over the four warps; red[buf] is rewritten two
      // blocks later, after thread 0 (which reads it) has arrived on d_free.
      ss = warp_sum(ss);
      if (lane == 0) {
        red[buf * 8 + warp] = ss;
        mbar_arrive(&red_full[buf]);
      }
      if (a == 0 && mbar_wait(&red_full[buf], (jj >> 1) & 1, abort))
        M[(size_t)bh * nb + j] = sqrtf(red[buf * 8] + red[buf * 8 + 1] + red[buf * 8 + 2] + red[buf * 8 + 3]);
      fence_before_sync();
      mbar_arrive(&d_free[buf]);
    }
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 5) tmem_dealloc(tmem, 256);
}

}  // namespace pisa
