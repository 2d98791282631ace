// Fused PISA forward on the 5th-generation tensor cores (bf16 inputs).
//
// gist.science technical summary of PISA, section 2: core algorithm (N_t
// equation, alpha_{t,j} = exp(q_t kbar_j^T)) and hardware implementation
// (phase 1: exact attention over the selected blocks; phase 2: zeroth-order
// scan over the unselected blocks' aggregated vectors; phase 3: the global
// first-order correction), all folded into ONE online softmax per row.
//
// Persistent CTAs, one per SM, walk "pairs" of consecutive 128-row query
// tiles (A, B) of one (batch, head), head-major so that the ~150 pairs in
// flight share one or two heads' K/V in L2.  Warp roles (384 threads; the
// softmax warpgroups raise their register limit to 200 with setmaxnreg, the
// third warpgroup drops to 104):
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: one thread per
//              query row (= TMEM lane).  Reads S, keeps the running max m, l =
//              D e^{-m} and beta e^{-m}, writes P (bf16) over S for the PV MMA,
//              rescales O in TMEM when m grows by more than 8 (log2 units;
//              exact since N and D carry the same factor), epilogue
//              o = (O + s beta q Hbar) / l.
//   warp 8     producer: streams Q tiles and a ring of 128-row operand tiles
//              with TMA, in the order of each pair's work list.
//   warp 9     MMA issuer: S = Q K^T and O += P V (P from TMEM), ping-ponging
//              the two tiles so that one tile's softmax overlaps the other
//              tile's MMAs.  The whole warp runs the issue loop and one
//              elected lane issues each instruction, which keeps the operands
//              in warp-uniform registers (a lone lane in a divergent branch
//              issues markedly slower).  Each step's ring items are taken
//              before the wait for P, and the PV and next-S groups go out back
//              to back.
//   warp 10    list builder: builds each pair's work list in shared memory
//              (two slots) one pair ahead of the other roles.
//   warp 11    idle.
// Work list of a pair: the exact KV blocks of each tile (for 64-token blocks a
// 128-row tile spans two query blocks: the union, with per-row-group bits),
// blocks selected by both tiles first and in the same order, so those K/V
// tiles are loaded once and feed both.  Every step covers 128 keys: one
// 128-token block, or two consecutive 64-token entries stacked in one ring
// slot (each 64-column half of S masked by its own entry), so the MMAs are
// always 128 x 128.  Then the centroid tiles (128 key
// centroids each, shared by both tiles, masked per tile), with the fp32
// centroid keys and value sums rounded to bf16: one MMA group each.  q_t Hbar
// (Hbar as a bf16 hi + lo pair) runs last into the tile's S columns.
//
// TMEM columns: [0,128) S_A, [128,256) S_B, [256,256+D) O_A, [256+D,256+2D) O_B.
#pragma once

#include "sm100.cuh"

namespace pisa {

struct FusedArgs {
  const int32_t* sel;
  __nv_bfloat16* out;
  int kk, L, nb, nbp, block;
  int n_qtiles;  // 128-row query tiles per (batch, head)
  int n_pairs;   // BH * ceil(n_qtiles / 2)
  float scale;       // 1/sqrt(d)
  float scale_log2;  // log2(e)/sqrt(d)
};

constexpr int kFusedThreads = 384;  // 3 warpgroups: softmax A, softmax B, producer/MMA
constexpr int kFusedStages = 4;

template <int D>
struct FusedLayout {
  static constexpr int QT = 128;
  static constexpr uint32_t kSlot = 128u * D * 2u;  // one operand tile
  static constexpr uint32_t kQ = QT * D * 2u;
  static constexpr uint32_t kRing = kFusedStages * kSlot;
  static constexpr int kNumBars = 2 * kFusedStages + 18;
  static constexpr uint32_t kBars = kNumBars * 8u;
  // one work-list slot: header[8] + entries A/B [G*kk each] + masks A/B [G*words each]
  __host__ __device__ static size_t list_ints(int G, int kk, int words) { return 8 + 2 * (size_t)G * kk + 2 * (size_t)G * words; }
  static size_t bytes(int G, int kk, int nbp) {
    return 1024 + 2 * kQ + kRing + kBars + 16 + 2 * 4 * list_ints(G, kk, nbp / 32);
  }
};

// Step structure of a pair, shared by the producer and the MMA issuer so that
// both walk the ring items in exactly the same order.
struct PairPlan {
  int nA, nB, nC, existsB, ncent;
  __device__ int U() const { return nA > nB ? nA : nB; }
  __device__ int T() const { return U() + ncent; }
  __device__ bool activeA(int u) const { return u < nA || u >= U(); }
  __device__ bool activeB(int u) const { return existsB && (u < nB || u >= U()); }
  __device__ bool shared(int u) const { return existsB && (u < nC || u >= U()); }
  __device__ bool centroid(int u) const { return u >= U(); }
};

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  return (static_cast<uint64_t>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

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
  constexpr uint32_t OC = 256;  // O_A at OC, O_B at OC + D

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;  // [2][kQ]
  uint8_t* sRing = smem + 2 * Lay::kQ;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRing + Lay::kRing);
  uint64_t* full = bars;
  uint64_t* empty = bars + NS;
  uint64_t* q_full = bars + 2 * NS;      // [2]
  uint64_t* q_empty = q_full + 2;        // [2]
  uint64_t* s_full = q_empty + 2;        // [2]
  uint64_t* p_full = s_full + 2;         // [2]
  uint64_t* o_final = p_full + 2;        // [2]
  uint64_t* epi_done = o_final + 2;      // [2]
  uint64_t* list_full = epi_done + 2;    // [2]
  uint64_t* list_empty = list_full + 2;  // [2]
  uint64_t* mma_idle = list_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Lay::kNumBars);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* lists = reinterpret_cast<int*>(tmem_slot + 4);
  const int words = a.nbp / 32;
  const int list_stride = (int)Lay::list_ints(G, a.kk, words);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nb = a.nb;
  const int n_cent = a.nbp / 128;
  const int pairs_per_head = (a.n_qtiles + 1) / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&q_full[x], 1);
      mbar_init(&q_empty[x], 1);
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 128);
      mbar_init(&o_final[x], 1);
      mbar_init(&epi_done[x], 128);
      mbar_init(&list_full[x], 1);
      mbar_init(&list_empty[x], 10);
    }
    mbar_init(mma_idle, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // Register split within the 384 x 168 registers the CTA is launched with:
  // the third warpgroup drops to 104, the softmax warpgroups rise to 200,
  // 2 x 128 x 200 + 128 x 104 = 64512 = 384 x 168 (an increase beyond the
  // launch total would wait forever).
  if (warp >= 8) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 104;\n" ::: "memory");
   if (warp == 10) {
    // ============================================================ list builder
    // Builds each pair's work list (header, entry lists, selection masks) one
    // pair ahead of the producer, the MMA issuer and the softmax warps, so that
    // none of them waits for it between pairs.
    bool ok = true;
    int lp = 0;
    for (int p = blockIdx.x; ok && p < a.n_pairs; p += gridDim.x, ++lp) {
      const int slot = lp & 1;
      int* L_ = lists + slot * list_stride;
      int* eA = L_ + 8;
      int* eB = eA + G * a.kk;
      uint32_t* mA = reinterpret_cast<uint32_t*>(eB + G * a.kk);
      uint32_t* mB = mA + G * words;
      if (!__all_sync(0xffffffffu, mbar_wait(&list_empty[slot], ((lp >> 1) & 1) ^ 1, abort))) {
        ok = false;
        break;
      }
      const int bh = p / pairs_per_head;
      const int tA = 2 * (p % pairs_per_head);
      const int existsB = (tA + 1) < a.n_qtiles;
      for (int e = lane; e < 2 * G * words; e += 32) mA[e] = 0u;
      __syncwarp();
      // Mask row r = x G + g is query block i = tA G + r; those rows are
      // consecutive in sel, so the pair's selections are one flat run of
      // n_sel entries.  Loads go out eight per lane before any atomic, so the
      // run costs a couple of L2 round trips, not one per 32 entries.
      {
        const int rows = min((1 + existsB) * G, nb - tA * G);
        const int n_sel = rows * a.kk;
        const int32_t* run = a.sel + ((size_t)bh * nb + (size_t)tA * G) * a.kk;
        for (int e0 = 0; e0 < n_sel; e0 += 32 * 8) {
          int jv[8];
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const int e = e0 + lane + 32 * m;
            jv[m] = e < n_sel ? __ldg(run + e) : 0;
          }
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const int e = e0 + lane + 32 * m;
            if (e >= n_sel) continue;
            const int j = jv[m];
            if (j < 0 || j >= nb) {
              raise_device_error(PISA_ERR_DEVICE_CHECK);
            } else {
              atomicOr(&mA[(e / a.kk) * words + (j >> 5)], 1u << (j & 31));
            }
          }
        }
      }
      __syncwarp();
      // Entry lists, all lanes: pass 0 the blocks of both tiles, pass 1 of A
      // only, pass 2 of B only, each ascending.  Lane l owns mask word w0 + l;
      // a warp scan of the words' bit counts gives each lane its output slot.
      int nA = 0, nB = 0, nC = 0;
      for (int pass = 0; pass < 3; ++pass) {
        for (int w0 = 0; w0 < words; w0 += 32) {
          const int w = w0 + lane;
          uint32_t bits = 0u;
          if (w < words) {
            uint32_t uA = 0, uB = 0;
#pragma unroll
            for (int g = 0; g < G; ++g) {
              uA |= mA[g * words + w];
              uB |= mB[g * words + w];
            }
            bits = pass == 0 ? (uA & uB) : pass == 1 ? (uA & ~uB) : (uB & ~uA);
          }
          const int c = __popc(bits);
          int incl = c;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          const int total = __shfl_sync(0xffffffffu, incl, 31);
          int pos = (pass == 2 ? nB : nA) + incl - c;
          while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1;
            int gA = 0, gB = 0;
#pragma unroll
            for (int g = 0; g < G; ++g) {
              gA |= ((mA[g * words + w] >> b) & 1u) << g;
              gB |= ((mB[g * words + w] >> b) & 1u) << g;
            }
            const int j = w * 32 + b;
            if (pass != 2) eA[pos] = j | (gA << 24);
            if (pass != 1) eB[pos] = j | (gB << 24);
            ++pos;
          }
          if (pass != 2) nA += total;
          if (pass != 1) nB += total;
          if (pass == 0) nC += total;
        }
      }
      __threadfence_block();
      __syncwarp();
      if (lane == 0) {
        // header: steps of A, B and shared steps (a step = 128 keys: one 128-token
        // block, or two consecutive list entries of 64 tokens), then the entry counts
        L_[0] = (nA + G - 1) / G;
        L_[1] = (nB + G - 1) / G;
        L_[2] = nC / G;
        L_[3] = existsB;
        L_[4] = bh;
        L_[5] = tA;
        L_[6] = nA;
        L_[7] = nB;
        // padding centroids [nb, nbp) count as selected in every mask, so the
        // softmax masks a centroid column with one bit test
        for (int w = nb >> 5; w < words; ++w) {
          const uint32_t pad = (w << 5) >= nb ? 0xffffffffu : ~((1u << (nb & 31)) - 1u);
          for (int g = 0; g < G; ++g) {
            mA[g * words + w] |= pad;
            mB[g * words + w] |= pad;
          }
        }
        mbar_arrive(&list_full[slot]);
      }
    }
   } else if (warp == 8) {
    // ================================================================ producer
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      prefetch_tensormap(&tmKc);
      prefetch_tensormap(&tmVc);
      prefetch_tensormap(&tmH);
    }
    int it = 0, qloads[2] = {0, 0};
    bool ok = true;
    int lp = 0;
    for (int p = blockIdx.x; ok && p < a.n_pairs; p += gridDim.x, ++lp) {
      const int slot = lp & 1;
      const int* L_ = lists + slot * list_stride;
      const int* eA = L_ + 8;
      const int* eB = eA + G * a.kk;
      if (!__all_sync(0xffffffffu, mbar_wait(&list_full[slot], (lp >> 1) & 1, abort))) {
        ok = false;
        break;
      }
      const int bh = p / pairs_per_head;
      const int tA = 2 * (p % pairs_per_head);
      const int existsB = (tA + 1) < a.n_qtiles;
      if (lane == 0) {
        const int nA = L_[6], nB = L_[7];  // entry counts
        const PairPlan pl{L_[0], L_[1], L_[2], L_[3], n_cent};
        // one ring item: `rows` rows at `row`, and when row2 >= 0 another `rows`
        // rows at row2 stacked below them (a 2 x 64-row step)
        auto load = [&](const CUtensorMap* map, int row, int rows, int row2) -> bool {
          const int s = it % NS;
          if (!mbar_wait(&empty[s], ((it / NS) & 1) ^ 1, abort)) return false;
          const int tile_rows = row2 >= 0 ? 2 * rows : rows;
          mbar_expect_tx(&full[s], tile_rows * D * 2);
#pragma unroll
          for (int cb = 0; cb < CB; ++cb) {
            uint8_t* dst = sRing + s * SLOT + cb * tile_rows * 128;
            tma_load_3d(dst, map, &full[s], cb * 64, row, bh);
            if (row2 >= 0) tma_load_3d(dst + rows * 128, map, &full[s], cb * 64, row2, bh);
          }
          ++it;
          return true;
        };
        // exact step u of tile x: entries G u .. G u + G - 1; a missing second
        // 64-token entry repeats the first (in bounds; its columns are masked)
        auto exact_item = [&](const CUtensorMap* map, int x, int u) -> bool {
          const int* e = x ? eB : eA;
          const int n = x ? nB : nA;
          const int j1 = e[G * u] & 0xFFFFFF;
          if (G == 1) return load(map, j1 * KB, KB, -1);
          const int j2 = (G * u + 1 < n) ? (e[G * u + 1] & 0xFFFFFF) : j1;
          return load(map, j1 * KB, KB, j2 * KB);
        };
        auto loadK = [&](int x, int u) -> bool {
          if (!pl.centroid(u)) return exact_item(&tmK, x, u);
          return load(&tmKc, (u - pl.U()) * 128, 128, -1);
        };
        auto loadV = [&](int x, int u) -> bool {
          if (!pl.centroid(u)) return exact_item(&tmV, x, u);
          return load(&tmVc, (u - pl.U()) * 128, 128, -1);
        };
        for (int x = 0; ok && x < 1 + existsB; ++x) {
          ok = mbar_wait(&q_empty[x], (qloads[x] & 1) ^ 1, abort);
          if (!ok) break;
          mbar_expect_tx(&q_full[x], Lay::kQ);
#pragma unroll
          for (int cb = 0; cb < CB; ++cb)
            tma_load_3d(sQ + x * Lay::kQ + cb * QT * 128, &tmQ, &q_full[x], cb * 64, (tA + x) * QT, bh);
          ++qloads[x];
        }
        const int T = pl.T();
        if (ok) ok = loadK(0, 0);
        if (ok && pl.activeB(0) && !pl.shared(0)) ok = loadK(1, 0);
        for (int u = 0; ok && u < T; ++u) {
          if (pl.activeA(u)) ok = loadV(0, u);
          if (ok && u + 1 < T && pl.activeA(u + 1)) ok = loadK(0, u + 1);
          if (ok && pl.activeB(u) && !pl.shared(u)) ok = loadV(1, u);
          if (ok && u + 1 < T && pl.activeB(u + 1) && !pl.shared(u + 1)) ok = loadK(1, u + 1);
        }
        if (ok) ok = load(&tmH, 0, D, -1) && load(&tmH, D, D, -1);
        // every copy of the pair is issued: the list is no longer read here
        if (ok) mbar_arrive(&list_empty[slot]);
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (lane == 0) {
      // the copies already issued land before the CTA can exit: the last load
      // of each ring slot (the latest phase of its full barrier) and the last
      // Q load of each tile buffer.  On the normal path the consumers have
      // seen them, or will; after another role gave up nothing else waits
      // for them.
      const int first = it > NS ? it - NS : 0;
      for (int u = first; u < it; ++u) mbar_drain(&full[u % NS], (u / NS) & 1);
      for (int x = 0; x < 2; ++x)
        if (qloads[x] > 0) mbar_drain(&q_full[x], (qloads[x] - 1) & 1);
    }
   } else if (warp == 9) {
    // ================================================================ MMA issuer
    // The whole warp runs the issue loop, so descriptors, slot indices and
    // barrier waits are warp-uniform; one elected lane issues each tcgen05
    // instruction.
    {
      constexpr uint32_t idC = idesc_bf16(128, 128, false, false);  // every step is 128 keys
      constexpr uint32_t idH = idesc_bf16(128, D, false, false);
      constexpr uint32_t idO = idesc_bf16(128, D, false, true);
      const uint32_t ring = smem_u32(sRing);
      const uint32_t qbase = smem_u32(sQ);
      auto qdesc = [&](int x, int kk) {
        return desc_sw128(qbase + x * Lay::kQ + (kk >> 2) * QT * 128 + (kk & 3) * 32, 16, 1024);
      };
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
      int qwaits[2] = {0, 0}, steps[2] = {0, 0}, epis[2] = {0, 0};
      bool ok = true;
      int lp = 0;
      for (int p = blockIdx.x; ok && p < a.n_pairs; p += gridDim.x, ++lp) {
        const int slot = lp & 1;
        if (!(ok = mbar_wait(&list_full[slot], (lp >> 1) & 1, abort))) break;
        const int* L_ = lists + slot * list_stride;
        const PairPlan pl{L_[0], L_[1], L_[2], L_[3], n_cent};
        const int T = pl.T();
        for (int x = 0; ok && x < 1 + pl.existsB; ++x) {
          ok = mbar_wait(&q_full[x], qwaits[x] & 1, abort);
          ++qwaits[x];
        }
        if (!ok) break;
        fence_after_sync();
        int ks = -1, vs = -1;  // slots of the last K / V items
        bool first_pv[2] = {true, true};
        auto s_mmas = [&](int x) {
          const uint32_t sc = tmem + x * 128;
          for (int kk = 0; kk < D / 16; ++kk) mma_ss_warp(sc, qdesc(x, kk), kdesc(ks, 128, kk), idC, kk > 0 ? 1u : 0u);
        };
        // Step u of tile x: O_x += P_x(u) V(u), then S_x = Q_x K(u+1)^T.  Both
        // ring items are taken before the wait for P, so their barrier waits
        // overlap the softmax instead of sitting between P and the next S; the
        // two MMA groups go out back to back and the commits follow them.  The
        // tensor pipe runs a CTA's MMAs in issue order, so S(u+1) overwrites
        // the S/P columns only after PV(u) has read P(u).
        auto issue_step = [&](int x, int u) -> bool {
          const bool pv = x == 0 ? pl.activeA(u) : pl.activeB(u);
          const bool sn = u + 1 < T && (x == 0 ? pl.activeA(u + 1) : pl.activeB(u + 1));
          // tile B reuses tile A's items on shared steps; tile A then keeps them
          if (pv && !((x == 1) && pl.shared(u)) && !take(vs)) return false;
          if (sn && !((x == 1) && pl.shared(u + 1)) && !take(ks)) return false;
          if (pv) {
            if (!mbar_wait(&p_full[x], steps[x] & 1, abort)) return false;
            ++steps[x];
            fence_after_sync();
            const uint32_t pa = tmem + x * 128;
            const uint32_t oc = tmem + OC + x * D;
            // one V item per step: a 128-token value tile or 128 centroid value sums
            for (int kk = 0; kk < 8; ++kk)
              mma_ts_warp(oc, pa + kk * 8, vdesc(vs, 128, kk), idO, (!first_pv[x] || kk > 0) ? 1u : 0u);
            first_pv[x] = false;
          }
          if (sn) s_mmas(x);
          if (pv && !((x == 0) && pl.shared(u))) mma_commit_warp(&empty[vs]);
          if (sn) {
            if (!((x == 0) && pl.shared(u + 1))) mma_commit_warp(&empty[ks]);
            mma_commit_warp(&s_full[x]);
          }
          return true;
        };
        // first S of a tile: before reusing S_x / O_x the previous epilogue of
        // tile x must have read them
        auto issue_first_s = [&](int x) -> bool {
          if (epis[x] > 0) {
            if (!mbar_wait(&epi_done[x], (epis[x] - 1) & 1, abort)) return false;
            fence_after_sync();
          }
          if (!((x == 1) && pl.shared(0)) && !take(ks)) return false;
          s_mmas(x);
          if (!((x == 0) && pl.shared(0))) mma_commit_warp(&empty[ks]);
          mma_commit_warp(&s_full[x]);
          return true;
        };
        ok = issue_first_s(0);
        if (ok && pl.activeB(0)) ok = issue_first_s(1);
        for (int u = 0; ok && u < T; ++u) {
          ok = issue_step(0, u);
          if (ok && pl.existsB) ok = issue_step(1, u);
        }
        if (!ok) break;
        // first-order term q Hbar into each tile's S columns; then Q and Hbar are free
        int h0, h1;
        if (!(ok = take(h0) && take(h1))) break;
        for (int x = 0; x < 1 + pl.existsB; ++x) {
          const uint32_t sc = tmem + x * 128;
          for (int kk = 0; kk < D / 16; ++kk) mma_ss_warp(sc, qdesc(x, kk), kdesc(h0, D, kk), idH, kk > 0 ? 1u : 0u);
          for (int kk = 0; kk < D / 16; ++kk) mma_ss_warp(sc, qdesc(x, kk), kdesc(h1, D, kk), idH, 1u);
          mma_commit_warp(&o_final[x]);
          mma_commit_warp(&q_empty[x]);
          ++epis[x];
        }
        mma_commit_warp(&empty[h0]);
        mma_commit_warp(&empty[h1]);
        if (lane == 0) mbar_arrive(&list_empty[slot]);
      }
      // every MMA issued (on the normal path too) completes before TMEM is freed
      mma_commit_warp(mma_idle);
      mbar_drain(mma_idle, 0);
    }
    __syncwarp();
   }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 200;\n" ::: "memory");
    // ================================================================ softmax: tile A (warps 0-3), B (4-7)
    const int x = warp / 4;
    const int row = threadIdx.x % 128;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp % 4) * 32) << 16);
    const uint32_t sbase = lane_base + x * 128;
    const uint32_t obase = lane_base + OC + x * D;
    const int g = row / KB;
    const float c2 = a.scale_log2;
    const int n_tail = a.L - (nb - 1) * a.block;
    int steps = 0, finals = 0;
    bool ok = true;
    int lp = 0;
    for (int p = blockIdx.x; ok && p < a.n_pairs; p += gridDim.x, ++lp) {
      const int slot = lp & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&list_full[slot], (lp >> 1) & 1, abort))) {
        ok = false;
        break;
      }
      const int* L_ = lists + slot * list_stride;
      const PairPlan pl{L_[0], L_[1], L_[2], L_[3], n_cent};
      const int bh = L_[4];
      const int qtile = L_[5] + x;
      const int* ent = L_ + 8 + x * G * a.kk;
      const int n_ent = L_[6 + x];
      int ent_win = -1, ent_reg = 0;
      const uint32_t* msk = reinterpret_cast<const uint32_t*>(L_ + 8 + 2 * G * a.kk) + x * G * words + g * words;
      if (x == 0 || pl.existsB) {
        const int qrow = qtile * QT + row;
        const int T = pl.T();
        float m = -INFINITY, l = 0.f, beta = 0.f;
        uint32_t s[128];
        for (int u = 0; u < T; ++u) {
          if (!(x == 0 ? pl.activeA(u) : pl.activeB(u))) continue;
          const bool exact = !pl.centroid(u);
          // Which keys of an exact step this row may use depends only on the
          // work list, so it is settled before the wait for S.  Column half h
          // (of KB columns) holds list entry G u + h: all of its tokens count if
          // the row's query block selected it, none otherwise (or when the
          // entry is absent).  The tile's list entries sit in a 32-entry
          // register window, one per lane, refilled every 32 entries.
          int nvalid[G];
          bool all_whole = false;
          // dead[h]: no row of this warp uses entry G u + h (its query block did
          // not select it): that half's P is zero without any exp2 (64-token
          // blocks only; a 128-token block is used by every row of the tile)
          bool dead[G];
#pragma unroll
          for (int h = 0; h < G; ++h) dead[h] = false;
          if (exact) {
            if (((G * u) >> 5) != ent_win) {
              ent_win = (G * u) >> 5;
              const int idx = ent_win * 32 + lane;
              ent_reg = idx < n_ent ? ent[idx] : 0;
            }
            bool whole = true;
#pragma unroll
            for (int h = 0; h < G; ++h) {
              nvalid[h] = 0;
              const int e = __shfl_sync(0xffffffffu, ent_reg, (G * u + h) & 31);
              if (G * u + h < n_ent) {
                const int j = e & 0xFFFFFF;
                if ((e >> (24 + g)) & 1) nvalid[h] = min(KB, a.L - j * KB);
              }
              whole = whole && nvalid[h] == KB;
              if (G > 1) dead[h] = __all_sync(0xffffffffu, nvalid[h] == 0);
            }
            all_whole = __all_sync(0xffffffffu, whole);
          }
          if (!__all_sync(0xffffffffu, mbar_wait(&s_full[x], steps & 1, abort))) {
            ok = false;
            break;
          }
          ++steps;
          fence_after_sync();
          float tmax = -INFINITY, x_tail = -INFINITY;
          tmem_ld32(sbase, s);
          tmem_ld32(sbase + 32, s + 32);
          tmem_ld32(sbase + 64, s + 64);
          tmem_ld32(sbase + 96, s + 96);
          tmem_wait_ld();
          if (exact) {
            if (all_whole) {
              float t0 = -INFINITY, t1 = -INFINITY, t2 = -INFINITY, t3 = -INFINITY;
#pragma unroll
              for (int c = 0; c < 128; c += 8) {
                t0 = fmax3(t0, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
                t1 = fmax3(t1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
                t2 = fmax3(t2, __uint_as_float(s[c + 4]), __uint_as_float(s[c + 5]));
                t3 = fmax3(t3, __uint_as_float(s[c + 6]), __uint_as_float(s[c + 7]));
              }
              tmax = fmax3(fmaxf(t0, t1), t2, t3);
            } else {
              // masked columns (an absent half, or past a ragged tail) become
              // -inf; four independent three-input max chains; a dead half is
              // skipped (its P is written as zero below)
              float t0 = -INFINITY, t1 = -INFINITY, t2 = -INFINITY, t3 = -INFINITY;
#pragma unroll
              for (int h = 0; h < G; ++h) {
                if (dead[h]) continue;
#pragma unroll
                for (int c = h * KB; c < h * KB + KB; c += 8) {
                  float v[8];
#pragma unroll
                  for (int e = 0; e < 8; ++e) {
                    const int cc = c + e;
                    v[e] = (cc % KB) < nvalid[h] ? __uint_as_float(s[cc]) : -INFINITY;
                    s[cc] = __float_as_uint(v[e]);
                  }
                  t0 = fmax3(t0, v[0], v[1]);
                  t1 = fmax3(t1, v[2], v[3]);
                  t2 = fmax3(t2, v[4], v[5]);
                  t3 = fmax3(t3, v[6], v[7]);
                }
              }
              tmax = fmax3(fmaxf(t0, t1), t2, t3);
            }
          } else {
            // centroid columns: masked when selected by this row's query block
            // (or padding); the mask words are the same for every row group
            // member, so the bit tests are uniform
            const int c0 = (u - pl.U()) * 128;
            const uint32_t* mw = msk + c0 / 32;
            const uint32_t bw[4] = {mw[0], mw[1], mw[2], mw[3]};
            // a partial tail block's centroid stands for n_tail tokens, not
            // block: read its logit before P overwrites S, to correct its mass
            const int ct = nb - 1 - c0;
            if (n_tail != a.block && ct >= 0 && ct < 128 && !((bw[ct >> 5] >> (ct & 31)) & 1u)) {
              x_tail = __uint_as_float(tmem_ld1(sbase + ct));
              tmem_wait_ld();
            }
            float t0 = -INFINITY, t1 = -INFINITY, t2 = -INFINITY, t3 = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; c += 8) {
              float v[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int cc = c + e;
                v[e] = ((bw[cc >> 5] >> (cc & 31)) & 1u) ? -INFINITY : __uint_as_float(s[cc]);
                s[cc] = __float_as_uint(v[e]);
              }
              t0 = fmax3(t0, v[0], v[1]);
              t1 = fmax3(t1, v[2], v[3]);
              t2 = fmax3(t2, v[4], v[5]);
              t3 = fmax3(t3, v[6], v[7]);
            }
            tmax = fmax3(fmaxf(t0, t1), t2, t3);
          }
          // running max in log2 units; lazy rescale when it grows by more than 8
          const float m_new = fmaxf(m, tmax * c2);
          float f = 1.f;
          if (m_new > m + 8.f) {
            if (m != -INFINITY) {
              f = ex2(m - m_new);
              l *= f;
              beta *= f;
            }
            m = m_new;
          }
          // O is quiescent here: this step's S MMA was issued after the previous
          // PV of this tile, so that PV has completed.
          if (__any_sync(0xffffffffu, f != 1.f)) {
            uint32_t o[32];
#pragma unroll 1
            for (int ch = 0; ch < D / 32; ++ch) {
              tmem_ld32(obase + ch * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
              tmem_st32(obase + ch * 32, o);
            }
            tmem_wait_st();
          }
          const float mu = (m == -INFINITY) ? 0.f : m;
          const uint64_t c2x2 = f2_pack(c2, c2), nmu = f2_pack(-mu, -mu);
          uint64_t acc = 0;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if (G > 1 && dead[hh * G / 2]) {
#pragma unroll
              for (int c = hh * 64; c < hh * 64 + 64; c += 2) s[c >> 1] = 0u;
            } else {
#pragma unroll
              for (int c = hh * 64; c < hh * 64 + 64; c += 2) {
                const uint64_t t = ffma2(f2_pack(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), c2x2, nmu);
                const float p0 = ex2(f2_lo(t));
                const float p1 = ex2(f2_hi(t));
                acc = fadd2(acc, f2_pack(p0, p1));
                s[c >> 1] = pack_bf16x2(p0, p1);
              }
            }
            if (hh == 0) tmem_st32(sbase, s);  // keys 0..63 go out while 64..127 are computed
          }
          const float sum = f2_lo(acc) + f2_hi(acc);
          if (exact) {
            l += sum;
          } else {
            beta += sum;
            l += (float)a.block * sum;
            if (x_tail != -INFINITY) l += (float)(n_tail - a.block) * ex2(x_tail * c2 - mu);
          }
          tmem_st32(sbase + 32, s + 32);
          tmem_wait_st();
          fence_before_sync();
          mbar_arrive(&p_full[x]);
        }
        if (!ok) break;
        // epilogue: o = (O + s beta q Hbar) / l, q Hbar in this tile's S columns
        if (!__all_sync(0xffffffffu, mbar_wait(&o_final[x], finals & 1, abort))) {
          ok = false;
          break;
        }
        ++finals;
        fence_after_sync();
        const float inv = 1.f / l;
        const float fo = a.scale * beta;
        __nv_bfloat16* dst = a.out + ((size_t)bh * a.L + qrow) * D;
#pragma unroll 1
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o[32], h[32];
          tmem_ld32(obase + ch * 32, o);
          tmem_ld32(sbase + ch * 32, h);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float y0 = fmaf(fo, __uint_as_float(h[2 * e]), __uint_as_float(o[2 * e])) * inv;
            const float y1 = fmaf(fo, __uint_as_float(h[2 * e + 1]), __uint_as_float(o[2 * e + 1])) * inv;
            pk[e] = pack_bf16x2(y0, y1);
          }
          if (qrow < a.L) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + ch * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
        }
        fence_before_sync();
        mbar_arrive(&epi_done[x]);
      }
      if (lane == 0) mbar_arrive(&list_empty[slot]);
    }
  }

  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 9) tmem_dealloc(tmem, 512);
}

// Centroid and Hbar operands of the fused kernel:
//   kc [BH][nbp][D]: bf16(kbar), zero padded
//   vc [BH][nbp][D]: bf16(value sums), zero padded
//   ht [BH][2*D][D]: Hbar transposed (row = value dim), bf16 hi then bf16 lo
// One bf16 per centroid statistic: the unselected blocks carry a small share
// of each row's softmax mass, so rounding kbar (in the exponent) and the value
// sums (in the numerator) to bf16 moves the output far less than the bf16
// output rounding itself (measured against the fp64 oracle on every parity
// shape).  Hbar keeps a hi + lo pair (two of ~1100 MMA groups per tile).
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
    const size_t dst = ((size_t)bh * nbp + j) * D + c;
    kc[dst] = kh;
    vc[dst] = vh;
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
