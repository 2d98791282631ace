// C ABI of the PISA library: argument validation, workspace carve-up and the
// launch sequence stats -> Hbar -> covariance norm -> routing -> fused forward.
// Every entry point validates on the host before any launch.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <type_traits>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "fused_simt.cuh"
#include "fused_sm100.cuh"
#include "route_variants.cuh"
#include "select.cuh"
#include "select_sm100.cuh"
#include "stats_simt.cuh"
#include "stats_sm100.cuh"

namespace pisa {
namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Shape {
  int batch, heads, L, d, block;
  int BH() const { return batch * heads; }
  int nb() const { return (L + block - 1) / block; }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// NVTX range around the launches of one stage (host-side enqueue; a profiler
// such as Nsight Systems lines it up with the kernels).  Without an attached
// tool the push and pop are no-op calls.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// ------------------------------------------------------------------ launch tuning
//
// Launch parameters that cannot change any result, chosen per (device, shape)
// by pisa_autotune or set explicitly; 0 means the built-in heuristic.
//   cov_j:      blocks per CTA of the covariance-norm kernel (each M_j comes
//               from its own block only)
//   select_r:   query blocks per CTA of the routing kernel (rows are scored
//               and selected independently)
//   fused_ctas: persistent CTAs of the fused kernel (each pair of query tiles
//               is computed by one CTA, whichever it is)
struct Tuning {
  int cov_j = 0, select_r = 0, fused_ctas = 0;
};
using TuneKey = std::tuple<int, int, int, int, int>;  // device, batch*heads, L, d, block
std::mutex g_tune_mutex;
std::map<TuneKey, Tuning> g_tune;

bool tune_key(int bh, int L, int d, int block, TuneKey* key) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  *key = TuneKey{dev, bh, L, d, block};
  return true;
}

Tuning tuning_for(int bh, int L, int d, int block) {
  TuneKey key;
  if (!tune_key(bh, L, d, block, &key)) return Tuning{};
  std::lock_guard<std::mutex> lock(g_tune_mutex);
  const auto it = g_tune.find(key);
  return it == g_tune.end() ? Tuning{} : it->second;
}

pisa_status check_shape(const Shape& s) {
  if (s.batch < 1 || s.heads < 1 || s.L < 1 || s.d < 1 || s.block < 1) return PISA_ERR_INVALID_ARG;
  if ((long long)s.batch * s.heads > 65535) return PISA_ERR_UNSUPPORTED;
  if (s.d != 64 && s.d != 128) return PISA_ERR_UNSUPPORTED;
  if (s.block != 64 && s.block != 128) return PISA_ERR_UNSUPPORTED;
  if ((long long)s.L * s.d * s.batch * s.heads > (1LL << 40)) return PISA_ERR_UNSUPPORTED;
  return PISA_OK;
}

template <typename... P>
bool all_ok(P... p) {
  const void* ptrs[] = {static_cast<const void*>(p)...};
  for (const void* x : ptrs)
    if (x == nullptr || !aligned16(x)) return false;
  return true;
}

// Blocks per CTA for the two streaming kernels (one CTA per SM: they use
// ~200 KB of shared memory).  A CTA's cost is its J blocks' input bytes plus a
// fixed overhead (pipeline fill and drain, about three blocks' worth of
// loads); the kernel's time follows the number of waves times that cost, so J
// minimises ceil(CTAs / 148) x (J x block_bytes + extra).  The B200's 148 SMs
// are a constant here so that workspace sizes do not depend on the device.
constexpr int kSMs = 148;

int wave_chunk(const Shape& s, long long block_bytes, long long extra, int jmin) {
  const long long bh = s.BH(), nb = s.nb();
  if (jmin < 1) jmin = 1;
  if (jmin > nb) jmin = (int)nb;
  long long best_cost = -1, best_j = jmin;
  for (long long J = jmin; J <= nb; ++J) {
    const long long ctas = bh * ((nb + J - 1) / J);
    const long long waves = (ctas + kSMs - 1) / kSMs;
    const long long cost = waves * (J * block_bytes + extra);
    if (best_cost < 0 || cost < best_cost || (cost == best_cost && J > best_j)) {
      best_cost = cost;
      best_j = J;
    }
  }
  return (int)best_j;
}

// Statistics kernel: reads q, k, v of each block (counted as bf16) and writes
// one d x d fp32 partial of Hbar per CTA; at least 2d / B blocks per CTA keep
// the partials under a third of the reads.
int stats_chunk(const Shape& s) {
  const long long in = 3LL * s.block * s.d * 2, ovh = 3LL * in;
  return wave_chunk(s, in, 4LL * s.d * s.d + ovh, (int)((2LL * s.d + s.block - 1) / s.block));
}
int stats_chunks(const Shape& s) {
  const int J = stats_chunk(s);
  return (s.nb() + J - 1) / J;
}

size_t stats_ws(const Shape& s) {
  return align_up((size_t)s.BH() * stats_chunks(s) * s.d * s.d * sizeof(float));
}

// bf16 operands of the tensor-core fused kernel: centroid keys [BH][nbp][d],
// value sums [BH][nbp][d], Hbar transposed as hi/lo [BH][2*d][d].
int padded_blocks(const Shape& s) { return (s.nb() + 127) / 128 * 128; }
size_t fused_ws(const Shape& s) {
  const size_t keys = align_up((size_t)s.BH() * padded_blocks(s) * s.d * 2);
  const size_t vals = align_up((size_t)s.BH() * padded_blocks(s) * s.d * 2);
  return keys + vals + align_up((size_t)s.BH() * 2 * s.d * s.d * 2);
}

struct Carve {
  float *qbar, *kbar, *vsum, *hbar, *M;
  int32_t* sel;
  void* stats;
  void* fused;
  size_t total;
};

Carve carve(const Shape& s, int k, char* base) {
  Carve c{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += align_up(bytes);
    return p;
  };
  const size_t stat = (size_t)s.BH() * s.nb() * s.d * sizeof(float);
  c.qbar = reinterpret_cast<float*>(take(stat));
  c.kbar = reinterpret_cast<float*>(take(stat));
  c.vsum = reinterpret_cast<float*>(take(stat));
  c.hbar = reinterpret_cast<float*>(take((size_t)s.BH() * s.d * s.d * sizeof(float)));
  c.M = reinterpret_cast<float*>(take((size_t)s.BH() * s.nb() * sizeof(float)));
  c.sel = reinterpret_cast<int32_t*>(take((size_t)s.BH() * s.nb() * k * sizeof(int32_t)));
  c.stats = take(stats_ws(s));
  c.fused = take(fused_ws(s));
  c.total = off;
  return c;
}

pisa_status last_launch() {
  return cudaGetLastError() == cudaSuccess ? PISA_OK : PISA_ERR_CUDA;
}

template <typename F>
bool set_smem(F* kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return true;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) ==
         cudaSuccess;
}

// ------------------------------------------------------------------ stages

bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer, uint32_t box_rows);

template <typename T, int D>
pisa_status run_stats(const T* q, const T* k, const T* v, const Shape& s, float* qbar, float* kbar,
                      float* vsum, float* hbar, float* partial, cudaStream_t st) {
  NvtxRange range("pisa.block_stats");
  const int J = stats_chunk(s), nc = stats_chunks(s);
  if constexpr (std::is_same<T, __nv_bfloat16>::value && D == 128) {
    CUtensorMap mQ, mK, mV;
    const uint32_t box = (uint32_t)s.block;
    if (!make_map(&mQ, q, D, s.L, s.BH(), box) || !make_map(&mK, k, D, s.L, s.BH(), box) ||
        !make_map(&mV, v, D, s.L, s.BH(), box))
      return PISA_ERR_CUDA;
    if (s.block == 128) {
      const size_t smem = StatsLayout<128>::bytes();
      if (!set_smem(stats_sm100_kernel<128>, smem)) return PISA_ERR_CUDA;
      stats_sm100_kernel<128><<<dim3(nc, s.BH()), kStatsThreads, smem, st>>>(mQ, mK, mV, s.L, s.nb(), J, qbar,
                                                                              kbar, vsum, partial);
    } else {
      const size_t smem = StatsLayout<64>::bytes();
      if (!set_smem(stats_sm100_kernel<64>, smem)) return PISA_ERR_CUDA;
      stats_sm100_kernel<64><<<dim3(nc, s.BH()), kStatsThreads, smem, st>>>(mQ, mK, mV, s.L, s.nb(), J, qbar,
                                                                            kbar, vsum, partial);
    }
    if (last_launch() != PISA_OK) return PISA_ERR_CUDA;
    hbar_reduce_kernel<D><<<dim3((D * D + 255) / 256, s.BH()), 256, 0, st>>>(partial, nc, s.nb(), hbar);
    return last_launch();
  }
  const size_t smem = (2 * (size_t)s.block * (D + 4) + 2 * D + 256) * sizeof(float);
  if (!set_smem(stats_simt_kernel<T, D>, smem)) return PISA_ERR_CUDA;
  stats_simt_kernel<T, D><<<dim3(nc, s.BH()), 256, smem, st>>>(q, k, v, s.L, s.block, s.nb(), J, qbar,
                                                                kbar, vsum, partial);
  if (last_launch() != PISA_OK) return PISA_ERR_CUDA;
  hbar_reduce_kernel<D><<<dim3((D * D + 255) / 256, s.BH()), 256, 0, st>>>(partial, nc, s.nb(), hbar);
  return last_launch();
}

// Covariance-norm kernel: reads k, v of each block; nothing per CTA but M.
int cov_chunk(const Shape& s) {
  const int tuned = tuning_for(s.BH(), s.L, s.d, s.block).cov_j;
  if (tuned > 0) return tuned < s.nb() ? tuned : s.nb();
  const long long in = 2LL * s.block * s.d * 2;
  return wave_chunk(s, in, 3LL * in, 1);
}

template <typename T, int D, bool WRITE_H>
pisa_status run_block_h(const T* k, const T* v, const Shape& s, const float* kbar, const float* vsum,
                        const float* hbar, float* out, cudaStream_t st) {
  NvtxRange range(WRITE_H ? "pisa.block_first_order" : "pisa.cov_norm");
  if constexpr (std::is_same<T, __nv_bfloat16>::value && D == 128 && !WRITE_H) {
    CUtensorMap mK, mV;
    const uint32_t box = (uint32_t)s.block;
    if (!make_map(&mK, k, D, s.L, s.BH(), box) || !make_map(&mV, v, D, s.L, s.BH(), box)) return PISA_ERR_CUDA;
    const int J = cov_chunk(s), nc = (s.nb() + J - 1) / J;
    if (s.block == 128) {
      const size_t smem = StatsLayout<128>::bytes();
      if (!set_smem(cov_norm_sm100_kernel<128>, smem)) return PISA_ERR_CUDA;
      cov_norm_sm100_kernel<128><<<dim3(nc, s.BH()), kStatsThreads, smem, st>>>(mK, mV, s.L, s.nb(), J, kbar, vsum,
                                                                                hbar, out);
    } else {
      const size_t smem = StatsLayout<64>::bytes();
      if (!set_smem(cov_norm_sm100_kernel<64>, smem)) return PISA_ERR_CUDA;
      cov_norm_sm100_kernel<64><<<dim3(nc, s.BH()), kStatsThreads, smem, st>>>(mK, mV, s.L, s.nb(), J, kbar, vsum,
                                                                               hbar, out);
    }
    return last_launch();
  }
  const size_t smem = (2 * (size_t)s.block * (D + 4) + 8) * sizeof(float);
  if (!set_smem(block_h_simt_kernel<T, D, WRITE_H>, smem)) return PISA_ERR_CUDA;
  block_h_simt_kernel<T, D, WRITE_H><<<dim3(s.nb(), s.BH()), 256, smem, st>>>(
      k, v, s.L, s.block, s.nb(), kbar, vsum, hbar, out);
  return last_launch();
}

// Routing on the tensor cores: R = 32 query blocks per CTA (the MMA's N), or
// 16 when the [R][nb] key buffer of 32 leaves no room for two 32 KB stages.
// Returns (R, stages), or R = 0 when even R = 16 does not fit (then the
// CUDA-core routing kernel, which needs no staging, takes the shape).
constexpr size_t kSmemMax = 227 * 1024;

template <int D, int R>
int select_tc_stages(int nb) {
  for (int ns = 4; ns >= 2; --ns)
    if (SelectTcLayout<D, R>::bytes(ns, nb) <= kSmemMax) return ns;
  return 0;
}

template <int D>
void select_tc_plan(int nb, int tuned_r, int* R, int* ns) {
  *R = 0;
  *ns = 0;
  const bool want16 = tuned_r > 0 && tuned_r <= 16;
  if (!want16 && (*ns = select_tc_stages<D, 32>(nb)) > 0) {
    *R = 32;
  } else if ((*ns = select_tc_stages<D, 16>(nb)) > 0) {
    *R = 16;
  }
}

// Largest routing tile of the CUDA-core kernel: R rows of nb keys in 140 KB, at most 32.
int select_rows_max(int nb) {
  // the key buffer (R x nb words) beside the fixed tiles, within 227 KB
  const long long budget = 140 * 1024;
  long long R = budget / (4LL * nb);
  if (R > 32) R = 32;
  return (int)R;
}

int select_rows(const Shape& s) {
  const int cap = select_rows_max(s.nb());
  const int tuned = tuning_for(s.BH(), s.L, s.d, s.block).select_r;
  return (tuned > 0 && tuned < cap) ? tuned : cap;
}

bool make_map_f32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer,
                  uint32_t box_rows);

template <int D, int R>
pisa_status launch_select_tc(const float* qbar, const float* kbar, const float* M, const Shape& s, int k,
                             int ns, int32_t* sel, cudaStream_t st) {
  const int nb = s.nb();
  CUtensorMap mK;
  if (!make_map_f32(&mK, kbar, D, nb, s.BH(), 128)) return PISA_ERR_CUDA;
  const size_t smem = SelectTcLayout<D, R>::bytes(ns, nb);
  if (!set_smem(select_sm100_kernel<D, R>, smem)) return PISA_ERR_CUDA;
  const float scale = 1.0f / sqrtf((float)D);
  const dim3 grid = (nb % R) != 0 ? dim3(s.BH(), (nb + R - 1) / R) : dim3((nb + R - 1) / R, s.BH());
  select_sm100_kernel<D, R><<<grid, kSelTcThreads, smem, st>>>(
      mK, qbar, M, s.L, s.block, nb, k, ns, scale, sel);
  return last_launch();
}

template <int D>
pisa_status run_select(const float* qbar, const float* kbar, const float* M, const Shape& s, int k,
                       int32_t* sel, cudaStream_t st) {
  NvtxRange range("pisa.select");
  const int nb = s.nb();
  int Rtc = 0, ns = 0;
  select_tc_plan<D>(nb, tuning_for(s.BH(), s.L, s.d, s.block).select_r, &Rtc, &ns);
  if (Rtc == 32) return launch_select_tc<D, 32>(qbar, kbar, M, s, k, ns, sel, st);
  if (Rtc == 16) return launch_select_tc<D, 16>(qbar, kbar, M, s, k, ns, sel, st);
  const int R = select_rows(s);
  if (R < 1) return PISA_ERR_UNSUPPORTED;
  const size_t smem = select_smem_bytes(D, R, nb);
  if (!set_smem(select_kernel<D>, smem)) return PISA_ERR_CUDA;
  const float scale = 1.0f / sqrtf((float)D);
  select_kernel<D><<<dim3((nb + R - 1) / R, s.BH()), kSelectThreads, smem, st>>>(qbar, kbar, M, s.L, s.block, nb,
                                                                      k, R, scale, sel);
  return last_launch();
}

template <typename T, int D>
pisa_status run_fused(const T* q, const T* k, const T* v, T* out, const Shape& s, const float* kbar,
                      const float* vsum, const float* hbar, const int32_t* sel, int kk,
                      cudaStream_t st) {
  NvtxRange range("pisa.fused");
  constexpr int TPR = 4, CH = 16, DS = D / TPR, RS = TPR * (DS + 4);
  const int nb = s.nb();
  const size_t smem = (2 * (size_t)CH * RS + (size_t)D * D + CH + (nb + 31) / 32) * sizeof(float);
  if (!set_smem(fused_simt_kernel<T, D, TPR, CH>, smem)) return PISA_ERR_CUDA;
  const float scale = 1.0f / sqrtf((float)D);
  fused_simt_kernel<T, D, TPR, CH><<<dim3(nb, s.BH()), s.block * TPR, smem, st>>>(
      q, k, v, out, s.L, s.block, nb, kk, kbar, vsum, hbar, sel, scale);
  return last_launch();
}

// The CUDA-core fused kernel with each unselected block's own first-order
// term (H: [BH][nb][D][D]), either dtype.
template <typename T, int D>
pisa_status run_fused_blockwise(const T* q, const T* k, const T* v, T* out, const Shape& s, const float* kbar,
                                const float* vsum, const float* H, const int32_t* sel, int kk, cudaStream_t st) {
  NvtxRange range("pisa.fused_blockwise");
  constexpr int TPR = 4, CH = 16, DS = D / TPR, RS = TPR * (DS + 4);
  const int nb = s.nb();
  const size_t smem = (2 * (size_t)CH * RS + (size_t)D * D + CH + (nb + 31) / 32) * sizeof(float);
  if (!set_smem(fused_simt_kernel<T, D, TPR, CH, true>, smem)) return PISA_ERR_CUDA;
  const float scale = 1.0f / sqrtf((float)D);
  fused_simt_kernel<T, D, TPR, CH, true><<<dim3(nb, s.BH()), s.block * TPR, smem, st>>>(
      q, k, v, out, s.L, s.block, nb, kk, kbar, vsum, H, sel, scale);
  return last_launch();
}

template <typename T, int D>
struct FusedBlockwiseOp {
  static pisa_status run(const void* q, const void* k, const void* v, void* out, const Shape& s,
                         const float* kbar, const float* vsum, const float* H, const int32_t* sel, int kk,
                         cudaStream_t st) {
    return run_fused_blockwise<T, D>((const T*)q, (const T*)k, (const T*)v, (T*)out, s, kbar, vsum, H, sel, kk,
                                     st);
  }
};

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  }
  return fn;
}

// 3-D bf16 map over [outer][rows][inner] with 64-element (128-byte) swizzled
// boxes of `box_rows` rows; reads outside [0, rows) return zeros.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer, uint32_t box_rows) {
  EncodeTiled fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {inner, rows, outer};
  const cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D fp32 map over [outer][rows][inner] with 32-element (128-byte) swizzled
// boxes of `box_rows` rows; reads outside [0, rows) return zeros.
bool make_map_f32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t outer,
                  uint32_t box_rows) {
  EncodeTiled fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {inner, rows, outer};
  const cuuint64_t strides[2] = {inner * 4, inner * rows * 4};
  const cuuint32_t box[3] = {32, box_rows, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int KB>
pisa_status run_fused_sm100(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                            __nv_bfloat16* out, const Shape& s, const float* kbar, const float* vsum,
                            const float* hbar, const int32_t* sel, int kk, void* ws, cudaStream_t st) {
  NvtxRange range("pisa.fused");
  const int nb = s.nb(), nbp = padded_blocks(s), BH = s.BH();
  char* w = static_cast<char*>(ws);
  const size_t keys = align_up((size_t)BH * nbp * D * 2);
  const size_t vals = align_up((size_t)BH * nbp * D * 2);
  __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(w);
  __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(w + keys);
  __nv_bfloat16* ht = reinterpret_cast<__nv_bfloat16*>(w + keys + vals);
  const int elems = nbp * D > D * D ? nbp * D : D * D;
  prep_fused_operands_kernel<D><<<dim3((elems + 255) / 256, BH), 256, 0, st>>>(kbar, vsum, hbar, nb, nbp, kc, vc, ht);
  if (last_launch() != PISA_OK) return PISA_ERR_CUDA;
  CUtensorMap mQ, mK, mV, mKc, mVc, mH;
  if (!make_map(&mQ, q, D, s.L, BH, 128) || !make_map(&mK, k, D, s.L, BH, KB) || !make_map(&mV, v, D, s.L, BH, KB) ||
      !make_map(&mKc, kc, D, nbp, BH, 128) || !make_map(&mVc, vc, D, nbp, BH, 128) ||
      !make_map(&mH, ht, D, 2 * D, BH, D))
    return PISA_ERR_CUDA;
  constexpr int G = 128 / KB;
  const size_t smem = FusedLayout<D>::bytes(G, kk, nbp);
  if (smem > 227 * 1024) return PISA_ERR_UNSUPPORTED;
  if (!set_smem(fused_sm100_kernel<D, KB>, smem)) return PISA_ERR_CUDA;
  FusedArgs fa;
  fa.sel = sel;
  fa.out = out;
  fa.kk = kk;
  fa.L = s.L;
  fa.nb = nb;
  fa.nbp = nbp;
  fa.block = s.block;
  fa.scale = 1.0f / sqrtf((float)D);
  fa.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  fa.n_qtiles = (s.L + 127) / 128;
  fa.n_pairs = BH * ((fa.n_qtiles + 1) / 2);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return PISA_ERR_CUDA;
  int grid = fa.n_pairs < sms ? fa.n_pairs : sms;
  const int tuned = tuning_for(s.BH(), s.L, s.d, s.block).fused_ctas;
  if (tuned > 0 && tuned < grid) grid = tuned;
  fused_sm100_kernel<D, KB><<<grid, kFusedThreads, smem, st>>>(mQ, mK, mV, mKc, mVc, mH, fa);
  return last_launch();
}

// dtype / d dispatch helpers
template <template <typename, int> class Op, typename... A>
pisa_status dispatch(pisa_dtype dt, int d, A&&... a) {
  if (dt == PISA_BF16) {
    if (d == 128) return Op<__nv_bfloat16, 128>::run(a...);
    if (d == 64) return Op<__nv_bfloat16, 64>::run(a...);
  } else if (dt == PISA_FP32) {
    if (d == 128) return Op<float, 128>::run(a...);
    if (d == 64) return Op<float, 64>::run(a...);
  }
  return PISA_ERR_UNSUPPORTED;
}

template <typename T, int D>
struct StatsOp {
  static pisa_status run(const void* q, const void* k, const void* v, const Shape& s, float* qbar,
                         float* kbar, float* vsum, float* hbar, float* partial, cudaStream_t st) {
    return run_stats<T, D>((const T*)q, (const T*)k, (const T*)v, s, qbar, kbar, vsum, hbar, partial, st);
  }
};

template <typename T, int D>
struct CovNormOp {
  static pisa_status run(const void* k, const void* v, const Shape& s, const float* kbar,
                         const float* vsum, const float* hbar, float* M, cudaStream_t st) {
    return run_block_h<T, D, false>((const T*)k, (const T*)v, s, kbar, vsum, hbar, M, st);
  }
};

template <typename T, int D>
struct FirstOrderOp {
  static pisa_status run(const void* k, const void* v, const Shape& s, const float* kbar,
                         const float* vsum, float* H, cudaStream_t st) {
    return run_block_h<T, D, true>((const T*)k, (const T*)v, s, kbar, vsum, nullptr, H, st);
  }
};

// fp32 inputs: CUDA-core fused kernel (tf32 MMAs cannot hold the fp32
// tolerance).  bf16 inputs: the tcgen05 tensor-core kernel.
template <typename T, int D>
struct FusedOp {
  static pisa_status run(const void* q, const void* k, const void* v, void* out, const Shape& s,
                         const float* kbar, const float* vsum, const float* hbar, const int32_t* sel,
                         int kk, void* ws, cudaStream_t st) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
      using B16 = __nv_bfloat16;
      if (s.block == 128)
        return run_fused_sm100<D, 128>((const B16*)q, (const B16*)k, (const B16*)v, (B16*)out, s, kbar, vsum,
                                       hbar, sel, kk, ws, st);
      return run_fused_sm100<D, 64>((const B16*)q, (const B16*)k, (const B16*)v, (B16*)out, s, kbar, vsum, hbar,
                                    sel, kk, ws, st);
    } else {
      (void)ws;
      return run_fused<T, D>((const T*)q, (const T*)k, (const T*)v, (T*)out, s, kbar, vsum, hbar, sel, kk, st);
    }
  }
};

bool valid_dtype(pisa_dtype dt) { return dt == PISA_BF16 || dt == PISA_FP32; }

}  // namespace

// Scratch of pisa_attn_fwd_with_sel_noalloc: one fixed device array per GPU
// that loads the library (held until the process exits).  Host code may not
// use the name as an address: the device address is looked up once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PISA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array for the current device; the first call
// on a device resolves it with that device current.
pisa_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PISA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return PISA_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return PISA_OK;
}
// The whole forward on device tensors of shape s (arguments already checked).
pisa_status forward_device(const void* q, const void* k, const void* v, void* out, pisa_dtype dtype,
                           const Shape& s, int kk, void* workspace, cudaStream_t st) {
  const Carve c = carve(s, kk, static_cast<char*>(workspace));
  const int d = s.d;
  pisa_status e = dispatch<StatsOp>(dtype, d, q, k, v, s, c.qbar, c.kbar, c.vsum, c.hbar, (float*)c.stats, st);
  if (e) return e;
  e = dispatch<CovNormOp>(dtype, d, k, v, s, (const float*)c.kbar, (const float*)c.vsum,
                          (const float*)c.hbar, c.M, st);
  if (e) return e;
  e = d == 128 ? run_select<128>(c.qbar, c.kbar, c.M, s, kk, c.sel, st)
               : run_select<64>(c.qbar, c.kbar, c.M, s, kk, c.sel, st);
  if (e) return e;
  return dispatch<FusedOp>(dtype, d, q, k, v, out, s, (const float*)c.kbar, (const float*)c.vsum,
                           (const float*)c.hbar, (const int32_t*)c.sel, kk, c.fused, st);
}

// ------------------------------------------------------------------ host-buffer forward
//
// Device workspace of pisa_attn_fwd_host: [forward scratch of one chunk]
// [slot 0: q, k, v, out of one chunk][slot 1: the same], each piece 256-byte
// aligned.  Sized for the widest element type (fp32) so one size query covers
// both dtypes.
struct HostPlan {
  int chunk;     // slices per chunk (clamped to batch*heads)
  size_t fwd;    // forward scratch: the larger of a full chunk's and the last chunk's
  size_t piece;  // one staged tensor of a full chunk
  size_t total() const { return align_up(fwd) + 8 * piece; }
  size_t slot_stride() const { return 4 * piece; }
};

HostPlan host_plan(const Shape& s, int kk, int chunk, pisa_dtype dtype) {
  HostPlan hp{};
  hp.chunk = chunk < s.BH() ? chunk : s.BH();
  const size_t es = dtype == PISA_BF16 ? 2 : 4;
  hp.piece = align_up((size_t)hp.chunk * s.L * s.d * es);
  // the stats scratch is not monotonic in the slice count, so size both chunk shapes that occur
  hp.fwd = carve(Shape{1, hp.chunk, s.L, s.d, s.block}, kk, nullptr).total;
  const int tail = s.BH() % hp.chunk;
  if (tail) {
    const size_t t = carve(Shape{1, tail, s.L, s.d, s.block}, kk, nullptr).total;
    if (t > hp.fwd) hp.fwd = t;
  }
  return hp;
}

// Per-device copy streams and events of the host-buffer forward, created on
// the first call on that device and kept until the process exits.
struct HostPipe {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, fin = nullptr;
  cudaEvent_t in_done[2] = {}, comp_done[2] = {}, out_done[2] = {};
};
std::mutex g_pipe_mutex;
HostPipe g_pipe[kMaxDevices];

pisa_status host_pipe(HostPipe** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PISA_ERR_CUDA;
  HostPipe& p = g_pipe[dev];
  if (!p.ready) {
    const unsigned ev = cudaEventDisableTiming;
    if (cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&p.start, ev) != cudaSuccess || cudaEventCreateWithFlags(&p.fin, ev) != cudaSuccess)
      return PISA_ERR_CUDA;
    for (int i = 0; i < 2; ++i)
      if (cudaEventCreateWithFlags(&p.in_done[i], ev) != cudaSuccess ||
          cudaEventCreateWithFlags(&p.comp_done[i], ev) != cudaSuccess ||
          cudaEventCreateWithFlags(&p.out_done[i], ev) != cudaSuccess)
        return PISA_ERR_CUDA;
    p.ready = true;
  }
  *out = &p;
  return PISA_OK;
}

pisa_status forward_host(const void* qh, const void* kh, const void* vh, void* oh, pisa_dtype dtype,
                         const Shape& s, int kk, const HostPlan& hp, char* ws, cudaStream_t st) {
  std::lock_guard<std::mutex> lock(g_pipe_mutex);
  HostPipe* p = nullptr;
  if (pisa_status e = host_pipe(&p)) return e;
  const size_t es = dtype == PISA_BF16 ? 2 : 4;
  const size_t slice = (size_t)s.L * s.d * es;
  char* fwd_ws = ws;
  char* slots = ws + align_up(hp.fwd);
  auto dev = [&](int slot, int t) { return slots + slot * hp.slot_stride() + t * hp.piece; };
  const char* src[3] = {static_cast<const char*>(qh), static_cast<const char*>(kh), static_cast<const char*>(vh)};
  char* dst = static_cast<char*>(oh);
  // copies start after the work already queued on the caller's stream (which
  // may still be using the workspace)
  if (cudaEventRecord(p->start, st) != cudaSuccess || cudaStreamWaitEvent(p->in, p->start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(p->out, p->start, 0) != cudaSuccess)
    return PISA_ERR_CUDA;
  const int BH = s.BH();
  for (int c = 0, first = 0; first < BH; ++c, first += hp.chunk) {
    const int n = BH - first < hp.chunk ? BH - first : hp.chunk;
    const int sl = c & 1;
    const size_t off = (size_t)first * slice, bytes = (size_t)n * slice;
    // inputs of this slot are free once the forward two chunks back has run
    if (c >= 2 && cudaStreamWaitEvent(p->in, p->comp_done[sl], 0) != cudaSuccess) return PISA_ERR_CUDA;
    for (int t = 0; t < 3; ++t)
      if (cudaMemcpyAsync(dev(sl, t), src[t] + off, bytes, cudaMemcpyHostToDevice, p->in) != cudaSuccess)
        return PISA_ERR_CUDA;
    if (cudaEventRecord(p->in_done[sl], p->in) != cudaSuccess) return PISA_ERR_CUDA;
    // the forward needs this chunk's inputs and an output slot already copied out
    if (cudaStreamWaitEvent(st, p->in_done[sl], 0) != cudaSuccess) return PISA_ERR_CUDA;
    if (c >= 2 && cudaStreamWaitEvent(st, p->out_done[sl], 0) != cudaSuccess) return PISA_ERR_CUDA;
    const Shape cs{1, n, s.L, s.d, s.block};
    if (pisa_status e = forward_device(dev(sl, 0), dev(sl, 1), dev(sl, 2), dev(sl, 3), dtype, cs, kk, fwd_ws, st))
      return e;
    if (cudaEventRecord(p->comp_done[sl], st) != cudaSuccess) return PISA_ERR_CUDA;
    if (cudaStreamWaitEvent(p->out, p->comp_done[sl], 0) != cudaSuccess ||
        cudaMemcpyAsync(dst + off, dev(sl, 3), bytes, cudaMemcpyDeviceToHost, p->out) != cudaSuccess ||
        cudaEventRecord(p->out_done[sl], p->out) != cudaSuccess)
      return PISA_ERR_CUDA;
  }
  // the caller's stream completes after the last output copy
  if (cudaEventRecord(p->fin, p->out) != cudaSuccess || cudaStreamWaitEvent(st, p->fin, 0) != cudaSuccess)
    return PISA_ERR_CUDA;
  return PISA_OK;
}
// Mean time of `reps` runs of fn on st (after one warm-up run), in ms.
template <typename F>
pisa_status time_on(cudaStream_t st, int reps, F fn, float* ms) {
  cudaEvent_t a, b;
  if (cudaEventCreate(&a) != cudaSuccess) return PISA_ERR_CUDA;
  if (cudaEventCreate(&b) != cudaSuccess) {
    cudaEventDestroy(a);
    return PISA_ERR_CUDA;
  }
  pisa_status e = fn();
  if (!e && cudaEventRecord(a, st) != cudaSuccess) e = PISA_ERR_CUDA;
  for (int r = 0; !e && r < reps; ++r) e = fn();
  if (!e && (cudaEventRecord(b, st) != cudaSuccess || cudaEventSynchronize(b) != cudaSuccess ||
             cudaEventElapsedTime(ms, a, b) != cudaSuccess))
    e = PISA_ERR_CUDA;
  if (!e) *ms /= reps;
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  return e;
}

void set_tuning(const TuneKey& key, const Tuning& t) {
  std::lock_guard<std::mutex> lock(g_tune_mutex);
  g_tune[key] = t;
}

// Tries each candidate of one parameter with the others fixed; keeps the fastest.
template <typename F>
pisa_status pick(const TuneKey& key, Tuning* t, int Tuning::*field, const int* cand, int n, cudaStream_t st,
                 F run) {
  float best_ms = 0.f;
  int best = 0;
  for (int c = 0; c < n; ++c) {
    Tuning trial = *t;
    trial.*field = cand[c];
    set_tuning(key, trial);
    float ms = 0.f;
    if (pisa_status e = time_on(st, 3, run, &ms)) return e;
    if (c == 0 || ms < best_ms) {
      best_ms = ms;
      best = cand[c];
    }
  }
  t->*field = best;
  set_tuning(key, *t);
  return PISA_OK;
}
}  // namespace
}  // namespace pisa

using namespace pisa;

extern "C" {

const char* pisa_status_string(pisa_status status) {
  switch (status) {
    case PISA_OK: return "ok";
    case PISA_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad size)";
    case PISA_ERR_UNSUPPORTED: return "unsupported shape (d and block must be 64 or 128)";
    case PISA_ERR_WORKSPACE: return "workspace missing or too small";
    case PISA_ERR_CUDA: return "CUDA runtime error";
    case PISA_ERR_TIMEOUT: return "a bounded device wait timed out";
    case PISA_ERR_DEVICE_CHECK: return "a device-side index check failed";
  }
  return "unknown status";
}

int pisa_keep_count(int L, int block, float keep_ratio) {
  if (L < 1 || block < 1 || !std::isfinite(keep_ratio) || keep_ratio <= 0.f) return -1;
  const long long nb = ((long long)L + block - 1) / block;
  long long k = (long long)std::ceil((double)keep_ratio * (double)nb - 1e-9);
  if (k < 1) k = 1;
  if (k > nb) k = nb;
  return (int)k;
}

size_t pisa_stats_workspace_size(int batch, int heads, int L, int d, int block) {
  const Shape s{batch, heads, L, d, block};
  if (check_shape(s) != PISA_OK) return 0;
  return stats_ws(s);
}

size_t pisa_fused_workspace_size(int batch, int heads, int L, int d, int block) {
  const Shape s{batch, heads, L, d, block};
  if (check_shape(s) != PISA_OK) return 0;
  return fused_ws(s);
}

size_t pisa_workspace_size(int batch, int heads, int L, int d, int block, int k) {
  const Shape s{batch, heads, L, d, block};
  if (check_shape(s) != PISA_OK || k < 1 || k > s.nb()) return 0;
  return carve(s, k, nullptr).total;
}

pisa_status pisa_block_stats(const void* q, const void* k, const void* v, pisa_dtype dtype, int batch,
                             int heads, int L, int d, int block, float* qbar, float* kbar, float* vsum,
                             float* hbar, void* workspace, size_t workspace_bytes, void* stream) {
  const Shape s{batch, heads, L, d, block};
  if (pisa_status e = check_shape(s)) return e;
  if (!valid_dtype(dtype)) return PISA_ERR_INVALID_ARG;
  if (!all_ok(q, k, v, qbar, kbar, vsum, hbar)) return PISA_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < stats_ws(s)) return PISA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return PISA_ERR_INVALID_ARG;
  return dispatch<StatsOp>(dtype, d, q, k, v, s, qbar, kbar, vsum, hbar, (float*)workspace,
                           (cudaStream_t)stream);
}

pisa_status pisa_cov_norm(const void* k, const void* v, pisa_dtype dtype, int batch, int heads, int L,
                          int d, int block, const float* kbar, const float* vsum, const float* hbar,
                          float* M, void* stream) {
  const Shape s{batch, heads, L, d, block};
  if (pisa_status e = check_shape(s)) return e;
  if (!valid_dtype(dtype)) return PISA_ERR_INVALID_ARG;
  if (!all_ok(k, v, kbar, vsum, hbar, M)) return PISA_ERR_INVALID_ARG;
  return dispatch<CovNormOp>(dtype, d, k, v, s, kbar, vsum, hbar, M, (cudaStream_t)stream);
}

pisa_status pisa_block_first_order(const void* k, const void* v, pisa_dtype dtype, int batch, int heads,
                                   int L, int d, int block, const float* kbar, const float* vsum,
                                   float* H, void* stream) {
  const Shape s{batch, heads, L, d, block};
  if (pisa_status e = check_shape(s)) return e;
  if (!valid_dtype(dtype)) return PISA_ERR_INVALID_ARG;
  if (!all_ok(k, v, kbar, vsum, H)) return PISA_ERR_INVALID_ARG;
  return dispatch<FirstOrderOp>(dtype, d, k, v, s, kbar, vsum, H, (cudaStream_t)stream);
}

pisa_status pisa_select(const float* qbar, const float* kbar, const float* M, int batch, int heads, int L,
                        int d, int block, int k, int32_t* sel, void* stream) {
  const Shape s{batch, heads, L, d, block};
  if (pisa_status e = check_shape(s)) return e;
  if (k < 1 || k > s.nb()) return PISA_ERR_INVALID_ARG;
  if (!all_ok(qbar, kbar, M) || sel == nullptr || (reinterpret_cast<uintptr_t>(sel) & 3u))
    return PISA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  return d == 128 ? run_select<128>(qbar, kbar, M, s, k, sel, st)
                  : run_select<64>(qbar, kbar, M, s, k, sel, st);
}

pisa_status pisa_select_route(const float* qbar, const float* kbar, const float* M, int batch, int heads, int L,
                              int d, int block, int k, pisa_route route, int32_t* sel, void* stream) {
  if (route == PISA_ROUTE_COVARIANCE) return pisa_select(qbar, kbar, M, batch, heads, L, d, block, k, sel, stream);
  if (route != PISA_ROUTE_POOLED) return PISA_ERR_INVALID_ARG;
  const Shape s{batch, heads, L, d, block};
  if (pisa_status e = check_shape(s)) return e;
  if (k < 1 || k > s.nb()) return PISA_ERR_INVALID_ARG;
  if (!all_ok(qbar, kbar) || sel == nullptr || (reinterpret_cast<uintptr_t>(sel) & 3u)) return PISA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  return d == 128 ? run_select<128>(qbar, kbar, nullptr, s, k, sel, st)
                  : run_select<64>(qbar, kbar, nullptr, s, k, sel, st);
}

pisa_status pisa_cov_norm_spectral(const float* H, const float* hbar, int batch, int heads, int L, int d,
                                   int block, float* M, void* stream) {
  const Shape s{batch, heads, L, d, block};
  if (pisa_status e = check_shape(s)) return e;
  if (!all_ok(H, hbar, M)) return PISA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (d == 128) {
    const size_t smem = (2 * 128 * 128 + 2 * 128 + 16) * sizeof(float);
    if (!set_smem(cov_spectral_kernel<128>, smem)) return PISA_ERR_CUDA;
    cov_spectral_kernel<128><<<dim3(s.nb(), s.BH()), kSpectralThreads, smem, st>>>(H, hbar, s.nb(), M);
  } else {
    const size_t smem = (2 * 64 * 64 + 2 * 64 + 16) * sizeof(float);
    if (!set_smem(cov_spectral_kernel<64>, smem)) return PISA_ERR_CUDA;
    cov_spectral_kernel<64><<<dim3(s.nb(), s.BH()), kSpectralThreads, smem, st>>>(H, hbar, s.nb(), M);
  }
  return last_launch();
}

pisa_status pisa_attn_fwd_with_sel(const void* q, const void* k, const void* v, void* out, pisa_dtype dtype,
                                   int batch, int heads, int L, int d, int block, const float* kbar,
                                   const float* vsum, const float* hbar, const int32_t* sel, int k_sel,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  const Shape s{batch, heads, L, d, block};
  if (pisa_status e = check_shape(s)) return e;
  if (!valid_dtype(dtype)) return PISA_ERR_INVALID_ARG;
  if (k_sel < 1 || k_sel > s.nb()) return PISA_ERR_INVALID_ARG;
  if (!all_ok(q, k, v, out, kbar, vsum, hbar) || sel == nullptr) return PISA_ERR_INVALID_ARG;
  if (dtype == PISA_BF16 && (workspace == nullptr || workspace_bytes < fused_ws(s))) return PISA_ERR_WORKSPACE;
  if (workspace != nullptr && !aligned16(workspace)) return PISA_ERR_INVALID_ARG;
  return dispatch<FusedOp>(dtype, d, q, k, v, out, s, kbar, vsum, hbar, sel, k_sel, workspace,
                           (cudaStream_t)stream);
}

pisa_status pisa_attn_fwd_blockwise_with_sel(const void* q, const void* k, const void* v, void* out,
                                             pisa_dtype dtype, int batch, int heads, int L, int d, int block,
                                             const float* kbar, const float* vsum, const float* H,
                                             const int32_t* sel, int k_sel, void* stream) {
  const Shape s{batch, heads, L, d, block};
  if (pisa_status e = check_shape(s)) return e;
  if (!valid_dtype(dtype)) return PISA_ERR_INVALID_ARG;
  if (k_sel < 1 || k_sel > s.nb()) return PISA_ERR_INVALID_ARG;
  if (!all_ok(q, k, v, out, kbar, vsum, H) || sel == nullptr) return PISA_ERR_INVALID_ARG;
  return dispatch<FusedBlockwiseOp>(dtype, d, q, k, v, out, s, kbar, vsum, H, sel, k_sel, (cudaStream_t)stream);
}

pisa_status pisa_attn_fwd_with_sel_noalloc(const void* q, const void* k, const void* v, void* out,
                                           pisa_dtype dtype, int batch, int heads, int L, int d, int block,
                                           const float* kbar, const float* vsum, const float* hbar,
                                           const int32_t* sel, int k_sel, void* stream) {
  const Shape s{batch, heads, L, d, block};
  if (pisa_status e = check_shape(s)) return e;
  if (!valid_dtype(dtype)) return PISA_ERR_INVALID_ARG;
  if (k_sel < 1 || k_sel > s.nb()) return PISA_ERR_INVALID_ARG;
  if (!all_ok(q, k, v, out, kbar, vsum, hbar) || sel == nullptr) return PISA_ERR_INVALID_ARG;
  // only the tensor-core (bf16) path takes scratch; the fp32 path uses none
  if (dtype == PISA_BF16 && fused_ws(s) > PISA_NOALLOC_SCRATCH_BYTES) return PISA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (pisa_status e = noalloc_scratch(&scratch)) return e;
  return dispatch<FusedOp>(dtype, d, q, k, v, out, s, kbar, vsum, hbar, sel, k_sel, scratch,
                           (cudaStream_t)stream);
}

pisa_status pisa_attn_fwd(const void* q, const void* k, const void* v, void* out, pisa_dtype dtype, int batch,
                          int heads, int L, int d, int block, float keep_ratio, void* workspace,
                          size_t workspace_bytes, void* stream) {
  const Shape s{batch, heads, L, d, block};
  if (pisa_status e = check_shape(s)) return e;
  if (!valid_dtype(dtype)) return PISA_ERR_INVALID_ARG;
  const int kk = pisa_keep_count(L, block, keep_ratio);
  if (kk < 1) return PISA_ERR_INVALID_ARG;
  if (!all_ok(q, k, v, out)) return PISA_ERR_INVALID_ARG;
  const Carve need = carve(s, kk, nullptr);
  if (workspace == nullptr || workspace_bytes < need.total) return PISA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return PISA_ERR_INVALID_ARG;
  return forward_device(q, k, v, out, dtype, s, kk, workspace, (cudaStream_t)stream);
}

size_t pisa_host_workspace_size(pisa_dtype dtype, int batch, int heads, int L, int d, int block, int k,
                                int chunk) {
  const Shape s{batch, heads, L, d, block};
  if (check_shape(s) != PISA_OK || !valid_dtype(dtype) || k < 1 || k > s.nb() || chunk < 1) return 0;
  return host_plan(s, k, chunk, dtype).total();
}

pisa_status pisa_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* out_host,
                               pisa_dtype dtype, int batch, int heads, int L, int d, int block,
                               float keep_ratio, int chunk, void* workspace, size_t workspace_bytes,
                               void* stream) {
  const Shape s{batch, heads, L, d, block};
  if (pisa_status e = check_shape(s)) return e;
  if (!valid_dtype(dtype)) return PISA_ERR_INVALID_ARG;
  const int kk = pisa_keep_count(L, block, keep_ratio);
  if (kk < 1 || chunk < 1) return PISA_ERR_INVALID_ARG;
  if (q_host == nullptr || k_host == nullptr || v_host == nullptr || out_host == nullptr)
    return PISA_ERR_INVALID_ARG;
  const HostPlan hp = host_plan(s, kk, chunk, dtype);
  if (workspace == nullptr || workspace_bytes < hp.total()) return PISA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return PISA_ERR_INVALID_ARG;
  return forward_host(q_host, k_host, v_host, out_host, dtype, s, kk, hp, static_cast<char*>(workspace),
                      (cudaStream_t)stream);
}

pisa_status pisa_autotune(const void* q, const void* k, const void* v, void* out, pisa_dtype dtype, int batch,
                          int heads, int L, int d, int block, float keep_ratio, void* workspace,
                          size_t workspace_bytes, void* stream, pisa_tuning* chosen) {
  const Shape s{batch, heads, L, d, block};
  if (pisa_status e = check_shape(s)) return e;
  if (!valid_dtype(dtype)) return PISA_ERR_INVALID_ARG;
  const int kk = pisa_keep_count(L, block, keep_ratio);
  if (kk < 1) return PISA_ERR_INVALID_ARG;
  if (!all_ok(q, k, v, out)) return PISA_ERR_INVALID_ARG;
  const Carve need = carve(s, kk, nullptr);
  if (workspace == nullptr || workspace_bytes < need.total) return PISA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return PISA_ERR_INVALID_ARG;
  TuneKey key;
  if (!tune_key(s.BH(), L, d, block, &key)) return PISA_ERR_CUDA;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return PISA_ERR_CUDA;
  const Carve c = carve(s, kk, static_cast<char*>(workspace));
  cudaStream_t st = (cudaStream_t)stream;
  Tuning t{};
  set_tuning(key, t);
  // inputs of the later stages: one default pass of stats and routing
  pisa_status e = dispatch<StatsOp>(dtype, d, q, k, v, s, c.qbar, c.kbar, c.vsum, c.hbar, (float*)c.stats, st);
  if (!e) e = dispatch<CovNormOp>(dtype, d, k, v, s, (const float*)c.kbar, (const float*)c.vsum,
                                  (const float*)c.hbar, c.M, st);
  if (!e) e = d == 128 ? run_select<128>(c.qbar, c.kbar, c.M, s, kk, c.sel, st)
                       : run_select<64>(c.qbar, c.kbar, c.M, s, kk, c.sel, st);
  if (e) return e;
  // covariance norm: blocks per CTA around the heuristic
  const int j0 = cov_chunk(s), nb = s.nb();
  int cj[4] = {j0, j0 > 1 ? j0 / 2 : 1, j0 * 2 < nb ? j0 * 2 : nb, j0 * 4 < nb ? j0 * 4 : nb};
  e = pick(key, &t, &Tuning::cov_j, cj, 4, st, [&] {
    return dispatch<CovNormOp>(dtype, d, k, v, s, (const float*)c.kbar, (const float*)c.vsum,
                               (const float*)c.hbar, c.M, st);
  });
  if (e) return e;
  // routing: rows per CTA; the tensor-core kernel runs 32 or 16 (the MMA's N),
  // the CUDA-core one up to what fits in shared memory
  int rtc = 0, ns = 0;
  if (d == 128) select_tc_plan<128>(nb, 0, &rtc, &ns); else select_tc_plan<64>(nb, 0, &rtc, &ns);
  const int rmax = select_rows_max(nb);
  int cr[4] = {rmax, rmax >= 24 ? 24 : rmax, rmax >= 16 ? 16 : rmax, rmax >= 8 ? 8 : rmax};
  const int ncr = rtc == 32 ? 2 : rtc == 16 ? 1 : 4;
  if (rtc > 0) {
    cr[0] = rtc;
    cr[1] = 16;
  }
  e = pick(key, &t, &Tuning::select_r, cr, ncr, st, [&] {
    return d == 128 ? run_select<128>(c.qbar, c.kbar, c.M, s, kk, c.sel, st)
                    : run_select<64>(c.qbar, c.kbar, c.M, s, kk, c.sel, st);
  });
  if (e) return e;
  // fused kernel: one CTA per SM, or the smallest grid with the same number of waves
  const long long pairs = (long long)s.BH() * ((((long long)L + 127) / 128 + 1) / 2);
  const long long waves = (pairs + sms - 1) / sms;
  const int balanced = (int)((pairs + waves - 1) / waves);
  int cf[3] = {sms, balanced < sms ? balanced : sms, sms - 4 > 0 ? sms - 4 : sms};
  e = pick(key, &t, &Tuning::fused_ctas, cf, 3, st, [&] {
    return dispatch<FusedOp>(dtype, d, q, k, v, out, s, (const float*)c.kbar, (const float*)c.vsum,
                             (const float*)c.hbar, (const int32_t*)c.sel, kk, c.fused, st);
  });
  if (e) return e;
  if (chosen) *chosen = pisa_tuning{t.cov_j, t.select_r, t.fused_ctas};
  return PISA_OK;
}

pisa_status pisa_set_tuning(int batch, int heads, int L, int d, int block, const pisa_tuning* t) {
  const Shape s{batch, heads, L, d, block};
  if (pisa_status e = check_shape(s)) return e;
  if (t && (t->cov_blocks_per_cta < 0 || t->select_rows_per_cta < 0 || t->select_rows_per_cta > 32 ||
            t->fused_ctas < 0))
    return PISA_ERR_INVALID_ARG;
  TuneKey key;
  if (!tune_key(s.BH(), L, d, block, &key)) return PISA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_tune_mutex);
  if (t == nullptr) {
    g_tune.erase(key);
  } else {
    g_tune[key] = Tuning{t->cov_blocks_per_cta, t->select_rows_per_cta, t->fused_ctas};
  }
  return PISA_OK;
}

pisa_status pisa_get_tuning(int batch, int heads, int L, int d, int block, pisa_tuning* t) {
  const Shape s{batch, heads, L, d, block};
  if (pisa_status e = check_shape(s)) return e;
  if (t == nullptr) return PISA_ERR_INVALID_ARG;
  const Tuning x = tuning_for(s.BH(), L, d, block);
  *t = pisa_tuning{x.cov_j, x.select_r, x.fused_ctas};
  return PISA_OK;
}

pisa_status pisa_tuning_save(const char* path) {
  if (path == nullptr) return PISA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return PISA_ERR_CUDA;
  FILE* f = std::fopen(path, "w");
  if (f == nullptr) return PISA_ERR_INVALID_ARG;
  std::fprintf(f, "# pisa launch tuning v1: batch*heads L d block cov_blocks_per_cta select_rows_per_cta fused_ctas\n");
  {
    std::lock_guard<std::mutex> lock(g_tune_mutex);
    for (const auto& kv : g_tune) {
      if (std::get<0>(kv.first) != dev) continue;
      std::fprintf(f, "%d %d %d %d %d %d %d\n", std::get<1>(kv.first), std::get<2>(kv.first),
                   std::get<3>(kv.first), std::get<4>(kv.first), kv.second.cov_j, kv.second.select_r,
                   kv.second.fused_ctas);
    }
  }
  return std::fclose(f) == 0 ? PISA_OK : PISA_ERR_INVALID_ARG;
}

pisa_status pisa_tuning_load(const char* path) {
  if (path == nullptr) return PISA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return PISA_ERR_CUDA;
  FILE* f = std::fopen(path, "r");
  if (f == nullptr) return PISA_ERR_INVALID_ARG;
  char line[256];
  pisa_status status = PISA_OK;
  std::map<TuneKey, Tuning> got;
  while (std::fgets(line, sizeof line, f)) {
    if (line[0] == '#' || line[0] == '\n') continue;
    int bh, L, d, block, cj, sr, fc;
    if (std::sscanf(line, "%d %d %d %d %d %d %d", &bh, &L, &d, &block, &cj, &sr, &fc) != 7 || bh < 1 ||
        check_shape(Shape{1, bh, L, d, block}) != PISA_OK || cj < 0 || sr < 0 || sr > 32 || fc < 0) {
      status = PISA_ERR_INVALID_ARG;
      break;
    }
    got[TuneKey{dev, bh, L, d, block}] = Tuning{cj, sr, fc};
  }
  std::fclose(f);
  if (status != PISA_OK) return status;  // a malformed file changes nothing
  std::lock_guard<std::mutex> lock(g_tune_mutex);
  for (const auto& kv : got) g_tune[kv.first] = kv.second;
  return PISA_OK;
}

pisa_status pisa_set_wait_limit(uint64_t limit_ns, void* stream) {
  const unsigned long long v = limit_ns == 0 ? kDefaultWaitLimitNs : (unsigned long long)limit_ns;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyToSymbolAsync(g_wait_limit_ns, &v, sizeof v, 0, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return PISA_ERR_CUDA;
  return PISA_OK;
}

pisa_status pisa_device_status(void* stream, int reset) {
  cudaStream_t st = (cudaStream_t)stream;
  int word = 0;
  if (cudaMemcpyFromSymbolAsync(&word, g_error_word, sizeof(int), 0, cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return PISA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PISA_ERR_CUDA;
  if (reset && word != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_error_word, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return PISA_ERR_CUDA;
  }
  if (word == 0) return PISA_OK;
  return (pisa_status)word;
}

}  // extern "C"
