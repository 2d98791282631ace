// Fused PISA forward on the 5th-generation tensor cores (bf16 inputs).
//
// gist.science technical summary of PISA, section 2: core algorithm (N_t
// equation, alpha_{t,j} = exp(q_t kbar_j^T)) and hardware implementation
// (phase 1: exact attention over the selected blocks; phase 2: zeroth-order
// scan over the unselected blocks' aggregated vectors; phase 3: the global
// first-order correction), all folded into ONE online softmax.
//
// One CTA per 128-row query tile of one (batch, head).  Warp roles:
//   warps 0-3  softmax: one thread per query row (= TMEM lane).  Reads S from
//              TMEM, keeps the running max m, l = D e^{-m}, beta e^{-m},
//              writes P (bf16) back over S for the PV MMA, rescales O in TMEM
//              when the max grows by more than 2^8 (lazy rescale; exact because
//              N and D carry the same factor), epilogue.
//   warp 4     TMA producer: Q once, then a ring of 128-row operand tiles.
//   warp 5     MMA issuer (one thread): S = Q K^T into a double-buffered TMEM
//              accumulator, O += P V with P read from TMEM.
// Tile sequence: the exact KV blocks of the tile's query block(s) (their
// union when a tile spans two 64-token blocks, with a per-row-group mask),
// then the centroid tiles (128 key centroids each; k and v are fp32 stats
// fed as bf16 hi + lo pairs, two MMAs each); the first-order term q_t Hbar
// (Hbar as hi + lo) is one more MMA into its own TMEM columns.
//
// TMEM columns: [0,128) S buffer 0, [128,256) S buffer 1, [256,256+D) O,
// [256+D, 256+2D) q Hbar.
#pragma once

#include "sm100.cuh"

namespace pisa {

struct FusedArgs {
  const int32_t* sel;
  __nv_bfloat16* out;
  int kk, L, nb, nbp, block;
  float scale;       // 1/sqrt(d)
  float scale_log2;  // log2(e)/sqrt(d)
};

constexpr int kFusedThreads = 192;
constexpr int kFusedStages = 4;

template <int D>
struct FusedLayout {
  static constexpr int QT = 128;
  static constexpr uint32_t kSlot = 128u * D * 2u;  // one operand tile
  static constexpr uint32_t kQ = QT * D * 2u;
  static constexpr uint32_t kRing = kFusedStages * kSlot;
  static constexpr uint32_t kBars = (2 * kFusedStages + 8) * 8u;
  static constexpr uint32_t kFixed = kQ + kRing + kBars + 16;
  // + list (G*kk ints) + masks (G * nbp/32 words), + 1024 alignment slack
  static size_t bytes(int G, int kk, int nbp) {
    return 1024 + kFixed + sizeof(int) * (size_t)G * kk + sizeof(uint32_t) * (size_t)G * (nbp / 32);
  }
};

template <int D, int KB>
__global__ void __launch_bounds__(kFusedThreads, 1)
fused_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKc,
                   const __grid_constant__ CUtensorMap tmVc, const __grid_constant__ CUtensorMap tmH,
                   const FusedArgs a) {
  using namespace sm100;
  using Lay = FusedLayout<D>;
  constexpr int QT = Lay::QT, G = QT / KB, CB = D / 64, NS = kFusedStages;
  constexpr uint32_t SLOT = Lay::kSlot;
  constexpr uint32_t OC = 256, QHC = 256 + D;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sRing = smem + Lay::kQ;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRing + Lay::kRing);
  uint64_t* full = bars;
  uint64_t* empty = bars + NS;
  uint64_t* q_full = bars + 2 * NS;
  uint64_t* s_full = q_full + 1;  // [2]
  uint64_t* p_full = s_full + 2;  // [2]
  uint64_t* o_done = p_full + 2;
  uint64_t* o_final = o_done + 1;
  uint64_t* mma_idle = o_final + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NS + 8);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* n_exact_s = reinterpret_cast<int*>(tmem_slot + 2);
  int* list = reinterpret_cast<int*>(tmem_slot + 4);
  const int words = a.nbp / 32;
  uint32_t* mask = reinterpret_cast<uint32_t*>(list + G * a.kk);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int qt = blockIdx.x, bh = blockIdx.y;
  const int nb = a.nb;

  // ------------------------------------------------------------ set-up
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&p_full[0], 128);
    mbar_init(&p_full[1], 128);
    mbar_init(o_done, 1);
    mbar_init(o_final, 1);
    mbar_init(mma_idle, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    prefetch_tensormap(&tmKc);
    prefetch_tensormap(&tmVc);
    prefetch_tensormap(&tmH);
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  for (int e = threadIdx.x; e < G * words; e += blockDim.x) mask[e] = 0u;
  __syncthreads();
  for (int g = 0; g < G; ++g) {
    const int i = qt * G + g;
    if (i >= nb) continue;
    const int32_t* si = a.sel + ((size_t)bh * nb + i) * a.kk;
    for (int e = threadIdx.x; e < a.kk; e += blockDim.x) {
      const int j = si[e];
      if (j < 0 || j >= nb) {
        raise_device_error(PISA_ERR_DEVICE_CHECK);
      } else {
        atomicOr(&mask[g * words + (j >> 5)], 1u << (j & 31));
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // exact tiles: ascending union of the selected blocks, with group bits
    int n = 0;
    for (int w = 0; w < words; ++w) {
      uint32_t any = 0;
#pragma unroll
      for (int g = 0; g < G; ++g) any |= mask[g * words + w];
      while (any) {
        const int b = __ffs(any) - 1;
        any &= any - 1;
        int gm = 0;
#pragma unroll
        for (int g = 0; g < G; ++g) gm |= ((mask[g * words + w] >> b) & 1u) << g;
        list[n++] = (w * 32 + b) | (gm << 24);
      }
    }
    *n_exact_s = n;
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int n_exact = *n_exact_s;
  const int n_cent = a.nbp / 128;
  const int n_t = n_exact + n_cent;

  if (warp == 4) {
    // -------------------------------------------------------- TMA producer
    if (lane == 0) {
      mbar_expect_tx(q_full, Lay::kQ);
#pragma unroll
      for (int cb = 0; cb < CB; ++cb) tma_load_3d(sQ + cb * QT * 128, &tmQ, q_full, cb * 64, qt * QT, bh);
      int it = 0;
      auto load = [&](const CUtensorMap* map, int row, int rows) -> bool {
        const int s = it % NS;
        const uint32_t ph = (it / NS) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, abort)) return false;
        mbar_expect_tx(&full[s], rows * D * 2);
#pragma unroll
        for (int cb = 0; cb < CB; ++cb) tma_load_3d(sRing + s * SLOT + cb * rows * 128, map, &full[s], cb * 64, row, bh);
        ++it;
        return true;
      };
      auto loadK = [&](int t) -> bool {
        if (t < n_exact) return load(&tmK, (list[t] & 0xFFFFFF) * KB, KB);
        const int c = t - n_exact;
        return load(&tmKc, c * 128, 128) && load(&tmKc, a.nbp + c * 128, 128);
      };
      auto loadV = [&](int t) -> bool {
        if (t < n_exact) return load(&tmV, (list[t] & 0xFFFFFF) * KB, KB);
        const int c = t - n_exact;
        return load(&tmVc, c * 128, 128) && load(&tmVc, a.nbp + c * 128, 128);
      };
      bool ok = load(&tmH, 0, D) && load(&tmH, D, D);
      for (int t = 0; ok && t < n_t; ++t) ok = loadK(t) && (t == 0 || loadV(t - 1));
      if (ok) ok = loadV(n_t - 1);
      if (!ok) {
        // let the copies already issued land before the CTA can exit
        const int first = it > NS ? it - NS : 0;
        for (int u = first; u < it; ++u) mbar_wait(&full[u % NS], (u / NS) & 1, abort);
      }
    }
  } else if (warp == 5) {
    // -------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, KB, false, false);
      constexpr uint32_t idC = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idH = idesc_bf16(128, D, false, false);
      constexpr uint32_t idO = idesc_bf16(128, D, false, true);
      const uint32_t qaddr = smem_u32(sQ);
      const uint32_t ring = smem_u32(sRing);
      auto qdesc = [&](int kk) { return desc_sw128(qaddr + (kk >> 2) * QT * 128 + (kk & 3) * 32, 16, 1024); };
      auto kdesc = [&](int s, int rows, int kk) {
        return desc_sw128(ring + s * SLOT + (kk >> 2) * rows * 128 + (kk & 3) * 32, 16, 1024);
      };
      auto vdesc = [&](int s, int rows, int kk) {
        return desc_sw128(ring + s * SLOT + kk * 16 * 128, rows * 128, 1024);
      };
      int it = 0;
      auto take = [&](int& s) -> bool {
        s = it % NS;
        if (!mbar_wait(&full[s], (it / NS) & 1, abort)) return false;
        fence_after_sync();
        ++it;
        return true;
      };
      auto pv = [&](int u) -> bool {
        const int buf = u & 1;
        if (!mbar_wait(&p_full[buf], (u >> 1) & 1, abort)) return false;
        fence_after_sync();
        const uint32_t pa = tmem + buf * 128;
        if (u < n_exact) {
          int s;
          if (!take(s)) return false;
          for (int kk = 0; kk < KB / 16; ++kk)
            mma_ts(tmem + OC, pa + kk * 8, vdesc(s, KB, kk), idO, (u > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&empty[s]);
        } else {
          int s1, s2;
          if (!take(s1) || !take(s2)) return false;
          for (int kk = 0; kk < 8; ++kk) mma_ts(tmem + OC, pa + kk * 8, vdesc(s1, 128, kk), idO, 1u);
          for (int kk = 0; kk < 8; ++kk) mma_ts(tmem + OC, pa + kk * 8, vdesc(s2, 128, kk), idO, 1u);
          mma_commit(&empty[s1]);
          mma_commit(&empty[s2]);
        }
        mma_commit(o_done);
        return true;
      };
      bool ok = mbar_wait(q_full, 0, abort);
      if (ok) {
        fence_after_sync();
        int sh, sl;
        ok = take(sh) && take(sl);
        if (ok) {
          for (int kk = 0; kk < D / 16; ++kk) mma_ss(tmem + QHC, qdesc(kk), kdesc(sh, D, kk), idH, kk > 0 ? 1u : 0u);
          for (int kk = 0; kk < D / 16; ++kk) mma_ss(tmem + QHC, qdesc(kk), kdesc(sl, D, kk), idH, 1u);
          mma_commit(&empty[sh]);
          mma_commit(&empty[sl]);
        }
      }
      for (int t = 0; ok && t < n_t; ++t) {
        const uint32_t sc = tmem + (t & 1) * 128;
        if (t < n_exact) {
          int s;
          ok = take(s);
          if (!ok) break;
          for (int kk = 0; kk < D / 16; ++kk) mma_ss(sc, qdesc(kk), kdesc(s, KB, kk), idS, kk > 0 ? 1u : 0u);
          mma_commit(&empty[s]);
        } else {
          int s1, s2;
          ok = take(s1) && take(s2);
          if (!ok) break;
          for (int kk = 0; kk < D / 16; ++kk) mma_ss(sc, qdesc(kk), kdesc(s1, 128, kk), idC, kk > 0 ? 1u : 0u);
          for (int kk = 0; kk < D / 16; ++kk) mma_ss(sc, qdesc(kk), kdesc(s2, 128, kk), idC, 1u);
          mma_commit(&empty[s1]);
          mma_commit(&empty[s2]);
        }
        mma_commit(&s_full[t & 1]);
        if (t >= 1) ok = pv(t - 1);
      }
      if (ok) ok = pv(n_t - 1);
      if (ok) mma_commit(o_final);
      // nothing of ours may still run on the tensor cores when TMEM is freed
      mma_commit(mma_idle);
      volatile int never = 0;
      mbar_wait(mma_idle, 0, &never);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------- softmax warps 0-3
    const int row = threadIdx.x;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int g = row / KB;
    const int qrow = qt * QT + row;
    const float c2 = a.scale_log2;
    const int n_tail = a.L - (nb - 1) * a.block;
    float m = -INFINITY, l = 0.f, beta = 0.f;
    uint32_t s[128];
    bool ok = true;
    for (int t = 0; t < n_t; ++t) {
      const int buf = t & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[buf], (t >> 1) & 1, abort))) {
        ok = false;
        break;
      }
      fence_after_sync();
      const uint32_t sa = lane_base + buf * 128;
      const bool exact = t < n_exact;
      float tmax = -INFINITY;
      float x_tail = -INFINITY;
      if (exact) {
        tmem_ld32(sa, s);
        if (KB == 128) {
          tmem_ld32(sa + 32, s + 32);
          tmem_ld32(sa + 64, s + 64);
          tmem_ld32(sa + 96, s + 96);
        } else {
          tmem_ld32(sa + 32, s + 32);
        }
        tmem_wait_ld();
        const int e = list[t];
        const int j = e & 0xFFFFFF;
        const int nvalid = ((e >> (24 + g)) & 1) ? min(KB, a.L - j * KB) : 0;
#pragma unroll
        for (int c = 0; c < KB; ++c) {
          const float x = c < nvalid ? __uint_as_float(s[c]) * c2 : -INFINITY;
          s[c] = __float_as_uint(x);
          tmax = fmaxf(tmax, x);
        }
      } else {
        tmem_ld32(sa, s);
        tmem_ld32(sa + 32, s + 32);
        tmem_ld32(sa + 64, s + 64);
        tmem_ld32(sa + 96, s + 96);
        tmem_wait_ld();
        const int c0 = (t - n_exact) * 128;
        const uint32_t* mw = mask + g * words + c0 / 32;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const uint32_t bits = mw[w];
#pragma unroll
          for (int b = 0; b < 32; ++b) {
            const int c = w * 32 + b;
            const bool use = (c0 + c < nb) && !((bits >> b) & 1u);
            const float x = use ? __uint_as_float(s[c]) * c2 : -INFINITY;
            s[c] = __float_as_uint(x);
            tmax = fmaxf(tmax, x);
            if (c0 + c == nb - 1) x_tail = x;
          }
        }
      }
      // lazy rescale: move the reference max only when it grows by > 2^8
      const float m_new = fmaxf(m, tmax);
      float f = 1.f;
      if (m_new > m + 8.f) {
        if (m != -INFINITY) {
          f = ex2(m - m_new);
          l *= f;
          beta *= f;
        }
        m = m_new;
      }
      const bool rescale_o = (f != 1.f) && t >= 1;
      if (__any_sync(0xffffffffu, rescale_o)) {
        if (!__all_sync(0xffffffffu, mbar_wait(o_done, (t - 1) & 1, abort))) {
          ok = false;
          break;
        }
        fence_after_sync();
        uint32_t o[32];
#pragma unroll 1
        for (int ch = 0; ch < D / 32; ++ch) {
          tmem_ld32(lane_base + OC + ch * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
          tmem_st32(lane_base + OC + ch * 32, o);
        }
        tmem_wait_st();
      }
      const float mu = (m == -INFINITY) ? 0.f : m;
      float sum = 0.f;
      const int ncols = exact ? KB : 128;
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        if (c < ncols) {
          const float p0 = ex2(__uint_as_float(s[c]) - mu);
          const float p1 = ex2(__uint_as_float(s[c + 1]) - mu);
          sum += p0 + p1;
          s[c >> 1] = pack_bf16x2(p0, p1);
        }
      }
      if (exact) {
        l += sum;
      } else {
        beta += sum;
        l += (float)a.block * sum;
        if (x_tail != -INFINITY) l += (float)(n_tail - a.block) * ex2(x_tail - mu);
      }
      tmem_st32(sa, s);
      if (ncols == 128) tmem_st32(sa + 32, s + 32);
      tmem_wait_st();
      fence_before_sync();
      mbar_arrive(&p_full[buf]);
    }
    // epilogue: o_t = (O + s beta q Hbar) / l
    if (ok && __all_sync(0xffffffffu, mbar_wait(o_final, 0, abort))) {
      fence_after_sync();
      const float inv = 1.f / l;
      const float fo = a.scale * beta;
      __nv_bfloat16* dst = a.out + ((size_t)bh * a.L + qrow) * D;
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32], h[32];
        tmem_ld32(lane_base + OC + ch * 32, o);
        tmem_ld32(lane_base + QHC + ch * 32, h);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float y0 = (__uint_as_float(o[2 * e]) + fo * __uint_as_float(h[2 * e])) * inv;
          const float y1 = (__uint_as_float(o[2 * e + 1]) + fo * __uint_as_float(h[2 * e + 1])) * inv;
          pk[e] = pack_bf16x2(y0, y1);
        }
        if (qrow < a.L) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + ch * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
    }
  }

  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 5) tmem_dealloc(tmem, 512);
}

// Centroid and Hbar operands in the fused kernel's bf16 hi/lo format:
//   kc [BH][2*nbp][D]: rows [0,nbp) bf16(kbar), rows [nbp,2nbp) bf16(kbar - hi); zero padded
//   vc [BH][2*nbp][D]: the same for the value sums
//   ht [BH][2*D][D]:   Hbar transposed (row = value dim), hi then lo
template <int D>
__global__ void prep_fused_operands_kernel(const float* __restrict__ kbar, const float* __restrict__ vsum,
                                           const float* __restrict__ hbar, int nb, int nbp,
                                           __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc,
                                           __nv_bfloat16* __restrict__ ht) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < nbp * D) {
    const int j = e / D, c = e % D;
    const size_t src = ((size_t)bh * nb + j) * D + c;
    const float kv = j < nb ? kbar[src] : 0.f;
    const float vv = j < nb ? vsum[src] : 0.f;
    const __nv_bfloat16 kh = __float2bfloat16_rn(kv), vh = __float2bfloat16_rn(vv);
    const size_t dst = ((size_t)bh * 2 * nbp + j) * D + c;
    kc[dst] = kh;
    kc[dst + (size_t)nbp * D] = __float2bfloat16_rn(kv - __bfloat162float(kh));
    vc[dst] = vh;
    vc[dst + (size_t)nbp * D] = __float2bfloat16_rn(vv - __bfloat162float(vh));
  }
  if (e < D * D) {
    const int c = e / D, r = e % D;  // ht[c][r] = Hbar[r][c]
    const float hv = hbar[(size_t)bh * D * D + (size_t)r * D + c];
    const __nv_bfloat16 hh = __float2bfloat16_rn(hv);
    const size_t dst = ((size_t)bh * 2 * D + c) * D + r;
    ht[dst] = hh;
    ht[dst + (size_t)D * D] = __float2bfloat16_rn(hv - __bfloat162float(hh));
  }
}

}  // namespace pisa
