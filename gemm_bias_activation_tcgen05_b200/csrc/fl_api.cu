// fl_api.cu — host side of the C ABI declared in include/fused_linear.h.
//
// fl_plan validates one layer ([epilog] page: Matmul(...).plan(epilog,
// epilog_inputs)), picks the kernel configuration for its shape and owns a
// tiny device workspace; fl_execute encodes the TMA descriptors for the
// caller's pointers and launches the fused kernel on the caller's stream
// ([epilog]: execute() is one kernel launch); fl_free releases the plan.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <new>

#include "../../include/fused_linear.h"
#include "fl_elementwise.cuh"
#include "fl_gemm.cuh"

using namespace fl;

// ------------------------------------------------------------------ errors
static thread_local char g_err[512] = "";
static uint64_t g_wait_limit_ns = 2000000000ull;

static fl_status fail(fl_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}
#define FL_CUDA(call)                                                                      \
  do {                                                                                     \
    cudaError_t e_ = (call);                                                               \
    if (e_ != cudaSuccess) return fail(FL_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

extern "C" const char* fl_last_error(void) { return g_err; }

extern "C" fl_status fl_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns = ns ? ns : 2000000000ull;
  return FL_OK;
}

// ------------------------------------------------------------------ driver entry point
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::once_flag g_encode_once;

static fl_status get_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return fail(FL_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  return FL_OK;
}

static int esize(int dt) { return dt == FL_F32 ? 4 : 2; }

// FL_SYNC_EACH_LAUNCH=1 (debug only): synchronise after every launch and name
// the launch whose execution failed.
static bool sync_each_launch() {
  static const bool on = [] {
    const char* v = getenv("FL_SYNC_EACH_LAUNCH");
    return v && v[0] == '1';
  }();
  return on;
}
static fl_status after_launch(cudaStream_t s, const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FL_ERR_CUDA, "%s: launch: %s", what, cudaGetErrorString(e));
  if (sync_each_launch()) {
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail(FL_ERR_CUDA, "%s: execution: %s", what, cudaGetErrorString(e));
  }
  return FL_OK;
}

static CUtensorMapDataType tm_dtype(int dt) {
  if (dt == FL_F32) return CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  if (dt == FL_BF16) return CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
}

// 2-D row-major map: `inner` contiguous elements per row, `outer` rows, row pitch in bytes.
static fl_status make_map(CUtensorMap* m, const void* base, int dt, uint64_t inner, uint64_t outer,
                          uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, tm_dtype(dt), 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(FL_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d): dims %llu x %llu pitch %llu box %u x %u",
                (int)r, (unsigned long long)inner, (unsigned long long)outer,
                (unsigned long long)pitch_bytes, box_inner, box_outer);
  return FL_OK;
}

// ------------------------------------------------------------------ kernel table
using KernelFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, KParams);

template <int ACT, int OUT>
static const void* pick_swap(bool swap) {
  return swap ? reinterpret_cast<const void*>(&fl_gemm_epi_tcgen05<ACT, OUT, true>)
              : reinterpret_cast<const void*>(&fl_gemm_epi_tcgen05<ACT, OUT, false>);
}
// fp32 operands (3xTF32): normal layout only
template <int ACT>
static const void* pick_tf32(int out) {
  if (out == FL_BF16) return reinterpret_cast<const void*>(&fl_gemm_epi_tcgen05<ACT, DT_BF16, false, true>);
  if (out == FL_F16) return reinterpret_cast<const void*>(&fl_gemm_epi_tcgen05<ACT, DT_F16, false, true>);
  return reinterpret_cast<const void*>(&fl_gemm_epi_tcgen05<ACT, DT_F32, false, true>);
}
template <int ACT>
static const void* pick_tf32_pair(int out) {
  if (out == FL_BF16) return reinterpret_cast<const void*>(&fl_gemm_epi_tcgen05<ACT, DT_BF16, false, true, true>);
  if (out == FL_F16) return reinterpret_cast<const void*>(&fl_gemm_epi_tcgen05<ACT, DT_F16, false, true, true>);
  return reinterpret_cast<const void*>(&fl_gemm_epi_tcgen05<ACT, DT_F32, false, true, true>);
}
static const void* pick_kernel_tf32_pair(int act, int out) {
  switch (act) {
    case ACT_NONE: return pick_tf32_pair<ACT_NONE>(out);
    case ACT_RELU: return pick_tf32_pair<ACT_RELU>(out);
    case ACT_GELU: return pick_tf32_pair<ACT_GELU>(out);
    case ACT_GELU_TANH: return pick_tf32_pair<ACT_GELU_TANH>(out);
    case ACT_GELU_SIGMOID: return pick_tf32_pair<ACT_GELU_SIGMOID>(out);
    default: return nullptr;
  }
}
static const void* pick_kernel_tf32(int act, int out) {
  switch (act) {
    case ACT_NONE: return pick_tf32<ACT_NONE>(out);
    case ACT_RELU: return pick_tf32<ACT_RELU>(out);
    case ACT_GELU: return pick_tf32<ACT_GELU>(out);
    case ACT_GELU_TANH: return pick_tf32<ACT_GELU_TANH>(out);
    case ACT_GELU_SIGMOID: return pick_tf32<ACT_GELU_SIGMOID>(out);
    default: return nullptr;
  }
}
template <int ACT>
static const void* pick_out(int out, bool swap) {
  if (out == FL_BF16) return pick_swap<ACT, DT_BF16>(swap);
  if (out == FL_F16) return pick_swap<ACT, DT_F16>(swap);
  return pick_swap<ACT, DT_F32>(swap);
}
// CTA-pair (256-row UMMA) kernels: normal layout, 16-bit operands
template <int ACT>
static const void* pick_pair(int out) {
  if (out == FL_BF16) return reinterpret_cast<const void*>(&fl_gemm_epi_tcgen05<ACT, DT_BF16, false, false, true>);
  if (out == FL_F16) return reinterpret_cast<const void*>(&fl_gemm_epi_tcgen05<ACT, DT_F16, false, false, true>);
  return reinterpret_cast<const void*>(&fl_gemm_epi_tcgen05<ACT, DT_F32, false, false, true>);
}
static const void* pick_kernel_pair(int act, int out) {
  switch (act) {
    case ACT_NONE: return pick_pair<ACT_NONE>(out);
    case ACT_RELU: return pick_pair<ACT_RELU>(out);
    case ACT_GELU: return pick_pair<ACT_GELU>(out);
    case ACT_GELU_TANH: return pick_pair<ACT_GELU_TANH>(out);
    case ACT_GELU_SIGMOID: return pick_pair<ACT_GELU_SIGMOID>(out);
    default: return pick_pair<ACT_GEGLU>(out);
  }
}
static const void* pick_kernel(int act, int out, bool swap) {
  switch (act) {
    case ACT_NONE: return pick_out<ACT_NONE>(out, swap);
    case ACT_RELU: return pick_out<ACT_RELU>(out, swap);
    case ACT_GELU: return pick_out<ACT_GELU>(out, swap);
    case ACT_GELU_TANH: return pick_out<ACT_GELU_TANH>(out, swap);
    case ACT_GELU_SIGMOID: return pick_out<ACT_GELU_SIGMOID>(out, swap);
    default: return swap ? nullptr : pick_out<ACT_GEGLU>(out, false);
  }
}

// ------------------------------------------------------------------ plan
// Tensor maps and kernel parameters of the last launch of one call site: a
// repeat call with the same operand pointers launches without re-encoding.
struct LaunchCache {
  bool valid = false;
  const void* key[8] = {};
  CUtensorMap tmA, tmB, tmB2, tmOut;
  KParams k;
};

struct fl_plan_s {
  int64_t M, N, K;
  int dtype, compute;
  fl_epilogue_desc epi;
  int act;
  bool has_bias, has_aux;
  int device, num_sms, max_smem;
  // configuration
  bool swap;
  bool pair;  // two CTAs share one 256-row UMMA tile (cluster of 2)
  int k_atoms;  // 128-byte K atoms per pipeline stage
  int mma_n, out_tile_n, split_k, stages, grid, smem;
  int tiles_a, tiles_b, num_kb;
  // stream-K (16-bit CTA pairs): the last sk_tiles tiles are split along K over
  // sk_clusters pairs; no_sk keeps the data-parallel schedule
  bool no_sk;
  int sk_tiles, sk_clusters;
  float* d_skws;  // partial accumulators, sk_ws_bytes()
  int* d_skflags;
  size_t skws_bytes, skflags_bytes;
  const void* kernel;
  int* d_err;
  // unfused twin
  void* d_tmp;
  int64_t tmp_ld;
  size_t tmp_bytes;
  int launches;
  uint64_t wait_limit_ns;
  LaunchCache cache_fused, cache_unfused;
};

static int act_of(int kind) {
  switch (kind) {
    case FL_EPI_RELU_BIAS:
    case FL_EPI_RELU_AUX_BIAS: return ACT_RELU;
    case FL_EPI_GELU_BIAS:
    case FL_EPI_GELU_AUX_BIAS: return ACT_GELU;
    case FL_EPI_GELU_TANH_BIAS: return ACT_GELU_TANH;
    case FL_EPI_GELU_SIGMOID_BIAS: return ACT_GELU_SIGMOID;
    case FL_EPI_GEGLU_TANH: return ACT_GEGLU;
    default: return ACT_NONE;
  }
}

static int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Shared-memory layout of one configuration: the operand ring, then (normal
// layout) the epilogue staging buffers and per-warp bias rows, then (split-K)
// the reduction buffer, then the barriers.
struct Layout {
  uint32_t a_stage, b_box, b_stage, stage, stride, staging_off, bias_off, bar_off, red_off, red_pitch, total;
  uint32_t res_off, res_blk;
  int stages;
};

constexpr int kMaxStages = 12;
static Layout layout_for(const fl_plan_s* p, int mma_n, int b_boxes, int max_smem) {
  Layout L{};
  const int es = esize(p->dtype);
  const int atoms = std::max(1, p->k_atoms);
  const int bk = atoms * 128 / es;
  const int rows_b = p->pair ? mma_n / 2 : mma_n;  // B rows (or columns) held by one CTA
  L.a_stage = (uint32_t)atoms * 128u * 128u;       // 128 rows x 128 bytes per atom
  if (p->epi.b_major) {
    L.b_box = 64u * (uint32_t)bk * (uint32_t)es;   // 64 columns x bk rows
    L.b_stage = L.b_box * (uint32_t)b_boxes;
  } else {
    L.b_box = (uint32_t)(rows_b / b_boxes) * 128u;
    L.b_stage = L.b_box * (uint32_t)b_boxes * (uint32_t)atoms;
  }
  L.stage = L.a_stage + L.b_stage;
  // fp32 operands: each stage also holds the TF32 lo halves of both tiles
  L.stride = (p->dtype == FL_F32) ? 2u * L.stage : L.stage;
  const uint32_t staging = p->swap ? Cfg<true>::kStagingBytes : Cfg<false>::kStagingBytes;
  const uint32_t bias = 0;
  // Split-K partial tiles (swap-AB, S > 1): a split-K cluster owns one tile, so the
  // partials are published after the last UMMA has read the last stage and can
  // reuse the stage memory.
  // (this CTA's partial, 128 rows, then S-1 received slices of 128/S rows each)
  const uint32_t red = (p->swap && p->split_k > 1)
                           ? (128u + (uint32_t)(p->split_k - 1) * (128u / (uint32_t)p->split_k)) *
                                 ((uint32_t)mma_n * 4u + 16u)
                           : 0u;
  // swap-AB with a residual: two 32-row x 32-column residual blocks per epilogue warp
  L.res_blk = 32u * 32u * (uint32_t)esize(p->epi.residual_dtype);
  const uint32_t res = (p->swap && p->epi.has_residual) ? (uint32_t)Cfg<true>::kEpiWarps * 2u * L.res_blk : 0u;
  const uint32_t bars = 8u * (3u * (uint32_t)kMaxStages + 8u);
  const uint32_t budget = (uint32_t)max_smem - 1024u - staging - bias - res - bars;
  int st = (int)(budget / L.stride);
  if (st > kMaxStages) st = kMaxStages;
  if (red > budget) st = 0;  // reported as "shared memory too small"
  L.stages = st;
  const uint32_t stage_area = std::max((uint32_t)st * L.stride, red);
  L.staging_off = stage_area;
  L.bias_off = L.staging_off + staging;
  L.red_off = 0;
  L.red_pitch = (uint32_t)mma_n * 4u + 16u;
  L.res_off = L.bias_off + bias;
  L.bar_off = L.res_off + res;
  L.total = L.bar_off + 8u * (3u * (uint32_t)st + 8u) + 1024u;
  return L;
}

// TMA boxes of operand B per stage and CTA.
static int b_boxes_of(const fl_plan_s* p, bool geglu) {
  const int rows_b = p->pair ? p->mma_n / 2 : p->mma_n;
  if (p->epi.b_major) return rows_b / 64;
  if (geglu) return p->pair ? 1 : 2;
  return 1;
}
static int grid_of(const fl_plan_s* p) {
  const int tiles = p->tiles_a * p->tiles_b;
  if (p->swap && p->split_k > 1) return tiles * p->split_k;
  // stream-K: every pair takes the same share of the full rounds and a range of the rest
  // (with fewer tiles than pairs, the 2·tiles pairs that share the tiles' K halves)
  if (p->pair && p->sk_tiles > 0) return 2 * std::max(p->sk_clusters, (tiles - p->sk_tiles > 0) ? p->num_sms / 2 : 0);
  if (p->pair) return 2 * std::min(tiles, p->num_sms / 2);
  return std::min(tiles, p->num_sms);
}
static const void* kernel_of(const fl_plan_s* p, int act, int out) {
  if (p->dtype == FL_F32) return p->pair ? pick_kernel_tf32_pair(act, out) : pick_kernel_tf32(act, out);
  if (p->pair) return pick_kernel_pair(act, out);
  return pick_kernel(act, out, p->swap);
}

// Stream-K for 16-bit CTA pairs.  Data-parallel, T tiles take ⌈T/P⌉ rounds of the P pairs.
// Stream-K spreads tiles over the pairs as contiguous ranges of (tile, K-block) units, at the
// price of a fix-up per cut tile: a 128 KB partial accumulator per CTA stored by the pair
// whose range starts inside the tile, then read and added by the pair holding the tile's
// first K blocks, before its epilogue.  The fix-up stays off the critical path when every
// range spans at least a whole tile: a writer stores its partial at the start of its range
// and the finisher adds it at the end of its own.  So:
//  * T > P: the tiles of the last, partial round plus one full round are split over all P
//    pairs (each range ≥ 1 tile, each cut tile split once); a pair saves
//    (⌈T/P⌉ − T/P)·num_kb K blocks;
//  * T ≤ P/2: each tile is split in two K halves over 2T pairs; a pair saves num_kb/2 K
//    blocks, and the finisher waits for the other half's store;
//  * otherwise (P/2 < T < P) the tiles stay whole.
// FL_SCHED_STREAM_K takes stream-K whenever one of the two forms applies.  FL_SCHED_AUTO keeps
// whole tiles: measured on a B200 (interleaved runs, CUDA-graph timed, 1965 MHz), stream-K
// tied or lost on every synthetic shape — 4096^3 119.2 vs 119.2 us, M = 2048 tail 84.8 vs
// 72.4, M = 512 tail 41.3 vs 39.0, GeGLU gate/up 84.8 vs 76.5 — except the GeGLU down
// projection (50.0 vs 51.2 us).  Even with the fix-up removed the stream-K ranges ran the
// main loop slower per K block than whole tiles do (M = 2048 tail: 79.2 vs 72.6 us).
static bool stream_k_pays(int64_t T, int64_t P, int num_kb, int schedule) {
  if (schedule != FL_SCHED_STREAM_K || num_kb < 2) return false;
  double saved;
  if (T > P) {
    if (T % P == 0) return false;
    saved = ((double)cdiv(T, P) - (double)T / (double)P) * num_kb;  // K blocks a pair saves
  } else if (2 * T <= P) {
    saved = (double)(num_kb / 2);
  } else {
    return false;
  }
  return saved > 0.0;
}

// The stream-K split of the chosen configuration (see stream_k_pays).
static void choose_stream_k(fl_plan_s* p) {
  p->sk_tiles = 0;
  p->sk_clusters = 0;
  if (!p->pair || p->no_sk || p->dtype == FL_F32) return;
  const int64_t P = p->num_sms / 2;
  const int64_t T = (int64_t)p->tiles_a * p->tiles_b;
  if (!stream_k_pays(T, P, p->num_kb, p->epi.schedule)) return;
  if (T > P) {
    p->sk_tiles = (int)(T % P + P);
    p->sk_clusters = (int)P;
  } else {
    p->sk_tiles = (int)T;
    p->sk_clusters = (int)(2 * T);
  }
}

static fl_status choose_config(fl_plan_s* p) {
  const int64_t M = p->M, N = p->N;
  const int es = esize(p->dtype);
  p->pair = false;
  const bool geglu = p->epi.kind == FL_EPI_GEGLU_TANH;
  // Small M: put the weight on the 128-row side of the tensor core (swap-AB)
  // and split K across a cluster so that every SM streams a slice of W.
  p->swap = (M <= 128) && !geglu && !p->epi.b_major && p->dtype != FL_F32;
  // Beyond one 128-row tile: CTA pairs with 256-row UMMA tiles.  16-bit operands take
  // 128-deep K stages (two swizzle atoms: eight UMMA steps per barrier round trip, and
  // 256 contiguous bytes of each operand row per stage, which the small-M layouts that
  // stream W from DRAM read faster than 128-byte pieces: measured on a B200, M = 32
  // tail 26.2 -> 22.6 us); fp32 operands keep one atom (a 3xTF32 stage also holds lo halves).
  p->pair = !p->swap && M > 128;
  p->k_atoms = (p->dtype != FL_F32) ? 2 : 1;
  p->num_kb = (int)cdiv(p->K, (int64_t)p->k_atoms * 128 / es);
  if (p->swap) {
    // The epilogue moves TMEM in 32-column chunks, so the activation tile is a multiple of 32.
    p->mma_n = (int)std::max<int64_t>(32, cdiv(M, 32) * 32);
    p->out_tile_n = p->mma_n;
    p->tiles_a = (int)cdiv(N, 128);
    p->tiles_b = (int)cdiv(M, p->mma_n);
    const int tiles = p->tiles_a * p->tiles_b;
    // split K over 1, 2 or 4 CTAs of a cluster (a reduce-scatter gives each CTA
    // 128/S output columns of the tile to finish)
    int S = 4;
    while (S > 1 && ((int64_t)tiles * S > p->num_sms || S > p->num_kb)) S >>= 1;
    p->split_k = S;
  } else {
    p->split_k = 1;
    const int rows = p->pair ? 256 : 128;
    const int units = p->pair ? p->num_sms / 2 : p->num_sms;
    if (geglu) {
      p->mma_n = 256;
      p->out_tile_n = 128;
    } else if (p->dtype == FL_F32 && !p->pair) {
      p->mma_n = 128;  // a 3xTF32 stage holds hi and lo tiles: 128 wide keeps three stages
      p->out_tile_n = 128;
    } else if (p->dtype == FL_F32) {
      // 3xTF32 pairs: the UMMA reads half of B from each CTA, halving the shared-memory
      // operand traffic per FLOP, which bounds this path.  Each epilogue warp covers
      // half the tile in chunks of 32 (fp32 out) or 64 (16-bit out) columns.
      const bool narrow_ok = esize(p->epi.out_dtype) == 4;
      int best = 256;
      double best_cost = 1e300;
      for (int bn : {256, 192, 128}) {
        if (bn == 192 && !narrow_ok) continue;
        const int64_t tiles = cdiv(M, rows) * cdiv(N, bn);
        const double waves = (double)cdiv(tiles, units);
        const double cost = waves * bn * (bn == 128 ? 1.3 : 1.0);
        if (cost < best_cost) { best_cost = cost; best = bn; }
      }
      p->mma_n = best;
      p->out_tile_n = best;
    } else {
      // Pick the N tile that minimises (waves x tile width) on this GPU.
      // Cost ~ (rounds of tiles per SM) x (tile width) x (relative cost per column):
      // narrower UMMA tiles move more operand bytes per FLOP and issue more instructions
      // per column; measured against 256 on a B200: 192 about 1.2-1.3x per column (a
      // 192-wide tile of a 16-bit output stores its warps' last 32 columns without TMA),
      // 128 about 1.5-1.6x.  With stream-K (CTA pairs) the rounds are fractional: the last,
      // partial round is spread over every pair.
      const bool sk_ok = p->pair && !p->no_sk;
      int best = 256;
      double best_cost = 1e300;
      for (int bn : {256, 192, 128}) {
        const int64_t tiles = cdiv(M, rows) * cdiv(N, bn);
        const bool sk = sk_ok && stream_k_pays(tiles, units, p->num_kb, p->epi.schedule);
        const double waves = sk ? (double)tiles / units : (double)cdiv(tiles, units);
        const double cost = waves * bn * (bn == 128 ? 1.6 : bn == 192 ? 1.25 : 1.0);
        if (cost < best_cost) { best_cost = cost; best = bn; }
      }
      p->mma_n = best;
      p->out_tile_n = best;
    }
    p->tiles_a = (int)cdiv(M, rows);
    p->tiles_b = (int)cdiv(N, p->out_tile_n);
    choose_stream_k(p);
  }
  return FL_OK;
}

// Stream-K workspace of a configuration: one fp32 partial accumulator per CTA and epilogue
// warp (mma_n/2 columns x 32 rows), and one flag per CTA and epilogue warp.
static void sk_sizes(const fl_plan_s* p, size_t* ws, size_t* flags) {
  *ws = *flags = 0;
  if (p->sk_tiles <= 0) return;
  *ws = (size_t)p->grid * 8u * (size_t)(p->mma_n / 2) * 32u * sizeof(float);
  *flags = (size_t)p->grid * 8u * sizeof(int);
}

// Configuration of the unfused twin's bare GEMM: the same operands with epilogue NONE,
// writing the [M, N] (GeGLU: [M, 2N]) intermediate.
static void twin_config(const fl_plan_s* p, fl_plan_s* q) {
  *q = *p;
  q->epi.kind = FL_EPI_NONE;
  q->epi.ldr = 0;
  q->epi.has_residual = 0;
  q->N = (p->epi.kind == FL_EPI_GEGLU_TANH) ? 2 * p->N : p->N;
  choose_config(q);
  const int b_boxes = b_boxes_of(q, false);
  Layout L = layout_for(q, q->mma_n, b_boxes, q->max_smem);
  q->stages = L.stages;
  q->smem = (int)L.total;
  q->grid = grid_of(q);
}

// Launches of one unfused execute: the bare GEMM, then one elementwise kernel per step.
static int unfused_launches(const fl_plan_s* p) {
  int steps = 0;
  if (p->epi.kind == FL_EPI_GEGLU_TANH) steps += 1;
  else steps += (p->has_bias ? 1 : 0) + (p->act != ACT_NONE ? 1 : 0);
  steps += (p->epi.has_residual ? 1 : 0) + (p->epi.scale != 1.0f ? 1 : 0);
  return 1 + steps;
}

// Everything fl_plan checks and records before it touches the device: the shape, the
// types, the epilogue descriptor and the row pitches.  On success *out is a new host
// plan (no device state yet) that the caller owns.
static fl_status plan_host_part(fl_plan_s** out, int64_t M, int64_t N, int64_t K, int32_t dtype, int32_t compute,
                                const fl_epilogue_desc* epi) {
  *out = nullptr;
  if (M < 1 || N < 1 || K < 0) return fail(FL_ERR_INVALID_ARG, "fl_plan: need M>=1, N>=1, K>=0 (got %lld %lld %lld)",
                                           (long long)M, (long long)N, (long long)K);
  if (M > (1LL << 31) - 256 || N > (1LL << 30) || K > (1LL << 31) - 256)
    return fail(FL_ERR_INVALID_ARG, "fl_plan: dimension too large");
  if (epi->kind < FL_EPI_NONE || epi->kind > FL_EPI_GELU_SIGMOID_BIAS)
    return fail(FL_ERR_INVALID_ARG, "fl_plan: unknown epilogue kind %d", epi->kind);
  for (int i = 0; i < 2; ++i)
    if (epi->reserved[i] != 0) return fail(FL_ERR_INVALID_ARG, "fl_plan: reserved fields must be 0");
  if (epi->schedule < FL_SCHED_AUTO || epi->schedule > FL_SCHED_STREAM_K)
    return fail(FL_ERR_INVALID_ARG, "fl_plan: unknown schedule %d", epi->schedule);
  if (dtype != FL_F16 && dtype != FL_BF16 && dtype != FL_F32)
    return fail(FL_ERR_INVALID_ARG, "fl_plan: unknown dtype %d", dtype);
  if (compute != FL_COMPUTE_32F && compute != FL_COMPUTE_32F_3XTF32)
    return fail(FL_ERR_UNSUPPORTED, "fl_plan: compute type %d not offered (only FP32 accumulation)", compute);
  if ((compute == FL_COMPUTE_32F) != (dtype != FL_F32))
    return fail(FL_ERR_UNSUPPORTED, "fl_plan: FL_COMPUTE_32F takes f16/bf16 operands, 3XTF32 takes f32");
  if (dtype == FL_F32 && (epi->b_major || epi->kind == FL_EPI_GEGLU_TANH))
    return fail(FL_ERR_UNSUPPORTED, "fl_plan: fp32 operands take a K-contiguous W and no GeGLU");
  if (epi->out_dtype < FL_F16 || epi->out_dtype > FL_F32)
    return fail(FL_ERR_INVALID_ARG, "fl_plan: unknown out_dtype %d", epi->out_dtype);
  const bool has_bias = epi->kind != FL_EPI_NONE && epi->kind != FL_EPI_GEGLU_TANH;
  if (has_bias && (epi->bias_dtype < FL_F16 || epi->bias_dtype > FL_F32))
    return fail(FL_ERR_INVALID_ARG, "fl_plan: unknown bias_dtype %d", epi->bias_dtype);
  if (epi->has_residual && (epi->residual_dtype < FL_F16 || epi->residual_dtype > FL_F32))
    return fail(FL_ERR_INVALID_ARG, "fl_plan: unknown residual_dtype %d", epi->residual_dtype);
  if (epi->bias_axis != 0 && epi->bias_axis != 1)
    return fail(FL_ERR_INVALID_ARG, "fl_plan: bias_axis must be 0 or 1");
  if (epi->b_major != 0 && epi->b_major != 1) return fail(FL_ERR_INVALID_ARG, "fl_plan: b_major must be 0 or 1");
  if (epi->kind == FL_EPI_GEGLU_TANH && epi->b_major)
    return fail(FL_ERR_UNSUPPORTED, "fl_plan: GEGLU_TANH takes the stacked [2N,K] weight (b_major 0)");
  if (epi->kind == FL_EPI_GEGLU_TANH && epi->out_dtype == FL_F32)
    return fail(FL_ERR_UNSUPPORTED, "fl_plan: GEGLU_TANH writes h in f16/bf16");
  if (epi->kind == FL_EPI_GELU_AUX_BIAS && epi->unfused)
    return fail(FL_ERR_UNSUPPORTED, "fl_plan: the unfused twin has no GELU_AUX_BIAS step");
  if (epi->lda < 0 || epi->ldb < 0 || epi->ldo < 0 || epi->ldr < 0)
    return fail(FL_ERR_INVALID_ARG, "fl_plan: negative leading dimension");

  fl_plan_s* p = new (std::nothrow) fl_plan_s();
  if (!p) return fail(FL_ERR_OOM, "fl_plan: host allocation failed");
  p->M = M; p->N = N; p->K = K; p->dtype = dtype; p->compute = compute; p->epi = *epi;
  if (p->epi.scale == 0.0f) p->epi.scale = 1.0f;
  p->act = act_of(epi->kind);
  p->has_bias = has_bias;
  p->has_aux = epi->kind == FL_EPI_RELU_AUX_BIAS || epi->kind == FL_EPI_GELU_AUX_BIAS;
  // leading dimensions default to packed
  const int64_t a_cols = K, b_cols = epi->b_major ? N : K;
  if (p->epi.lda == 0) p->epi.lda = a_cols;
  if (p->epi.ldb == 0) p->epi.ldb = b_cols;
  if (p->epi.ldo == 0) p->epi.ldo = N;
  if (p->epi.ldr == 0) p->epi.ldr = N;
  if (p->epi.lda < a_cols || p->epi.ldb < b_cols || p->epi.ldo < N || (epi->has_residual && p->epi.ldr < N)) {
    delete p;
    return fail(FL_ERR_INVALID_ARG, "fl_plan: leading dimension smaller than the row length");
  }
  const int es = esize(dtype), eo = esize(epi->out_dtype);
  if ((p->epi.lda * es) % 16 || (p->epi.ldb * es) % 16 || (p->epi.ldo * eo) % 16 ||
      (epi->has_residual && (p->epi.ldr * esize(epi->residual_dtype)) % 16)) {
    delete p;
    return fail(FL_ERR_ALIGNMENT, "fl_plan: every row pitch must be a multiple of 16 bytes");
  }
  *out = p;
  return FL_OK;
}

extern "C" fl_status fl_plan(fl_plan_t* out, int64_t M, int64_t N, int64_t K, int32_t dtype,
                             int32_t compute, const fl_epilogue_desc* epi) {
  g_err[0] = 0;
  if (!out || !epi) return fail(FL_ERR_INVALID_ARG, "fl_plan: null out or epilogue descriptor");
  *out = nullptr;
  fl_plan_s* p = nullptr;
  {
    const fl_status st0 = plan_host_part(&p, M, N, K, dtype, compute, epi);
    if (st0 != FL_OK) return st0;
  }
  const int eo = esize(epi->out_dtype);

  if (cudaGetDevice(&p->device) != cudaSuccess) { delete p; return fail(FL_ERR_DEVICE, "fl_plan: no CUDA device"); }
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, p->device) != cudaSuccess) {
    delete p;
    return fail(FL_ERR_DEVICE, "fl_plan: cannot query the device");
  }
  if (prop.major != 10) {
    delete p;
    return fail(FL_ERR_DEVICE, "fl_plan: needs an sm_100 (B200-class) GPU, found sm_%d%d", prop.major, prop.minor);
  }
  p->num_sms = prop.multiProcessorCount;
  p->max_smem = (int)prop.sharedMemPerBlockOptin;
  fl_status st = get_encode();
  if (st != FL_OK) { delete p; return st; }

  choose_config(p);
  const int b_boxes = b_boxes_of(p, p->epi.kind == FL_EPI_GEGLU_TANH);
  Layout L = layout_for(p, p->mma_n, b_boxes, p->max_smem);
  if (L.stages < 2) { delete p; return fail(FL_ERR_UNSUPPORTED, "fl_plan: shared memory too small"); }
  p->stages = L.stages;
  p->smem = (int)L.total;
  p->grid = grid_of(p);
  p->kernel = kernel_of(p, p->act, epi->out_dtype);
  if (!p->kernel) { delete p; return fail(FL_ERR_UNSUPPORTED, "fl_plan: no kernel for this combination"); }
  // Every plan sharing a kernel may need a different amount of dynamic shared
  // memory, so the kernel's bound is the device maximum, not this plan's size.
  cudaError_t e = cudaFuncSetAttribute(p->kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, p->max_smem);
  if (e != cudaSuccess) { delete p; return fail(FL_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e)); }
  if (p->split_k > 1) {
    e = cudaFuncSetAttribute(p->kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
    (void)e;
  }
  if (cudaMalloc(&p->d_err, sizeof(int)) != cudaSuccess) { delete p; return fail(FL_ERR_OOM, "fl_plan: cudaMalloc(error word)"); }
  if (cudaMemset(p->d_err, 0, sizeof(int)) != cudaSuccess) {
    cudaFree(p->d_err);
    delete p;
    return fail(FL_ERR_CUDA, "fl_plan: cudaMemset(error word)");
  }
  p->launches = 1;
  p->wait_limit_ns = g_wait_limit_ns;
  {
    // stream-K workspace: for this plan's kernel, and for the unfused twin's bare GEMM
    size_t ws = 0, fb = 0;
    sk_sizes(p, &ws, &fb);
    if (epi->unfused) {
      fl_plan_s q;
      twin_config(p, &q);
      size_t ws2 = 0, fb2 = 0;
      sk_sizes(&q, &ws2, &fb2);
      ws = std::max(ws, ws2);
      fb = std::max(fb, fb2);
    }
    if (ws > 0) {
      if (cudaMalloc(&p->d_skws, ws) != cudaSuccess || cudaMalloc(&p->d_skflags, fb) != cudaSuccess) {
        (void)cudaGetLastError();
        fl_free(p);
        return fail(FL_ERR_OOM, "fl_plan: cudaMalloc(stream-K workspace, %zu bytes)", ws + fb);
      }
      if (cudaMemset(p->d_skflags, 0, fb) != cudaSuccess) {
        fl_free(p);
        return fail(FL_ERR_CUDA, "fl_plan: cudaMemset(stream-K flags)");
      }
      p->skws_bytes = ws;
      p->skflags_bytes = fb;
    }
  }
  if (epi->unfused) {
    // the bare GEMM kernels of both layouts may serve this plan's first step
    for (int sw = 0; sw < 3; ++sw) {
      const void* kn = (dtype == FL_F32) ? (sw == 2 ? pick_kernel_tf32_pair(ACT_NONE, epi->out_dtype)
                                                    : pick_kernel_tf32(ACT_NONE, epi->out_dtype))
                       : (sw == 2 ? pick_kernel_pair(ACT_NONE, epi->out_dtype)
                                  : pick_kernel(ACT_NONE, epi->out_dtype, sw == 1));
      if (cudaFuncSetAttribute(kn, cudaFuncAttributeMaxDynamicSharedMemorySize, p->max_smem) != cudaSuccess) {
        cudaFree(p->d_err);
        delete p;
        return fail(FL_ERR_CUDA, "cudaFuncSetAttribute (unfused GEMM)");
      }
    }
    p->launches = unfused_launches(p);
    // GEMM into a plan-owned intermediate (the [M, N] or [M, 2N] result), then one
    // elementwise kernel per epilogue step.
    const int64_t cols = (epi->kind == FL_EPI_GEGLU_TANH) ? 2 * N : N;
    p->tmp_ld = cdiv(cols * eo, 16) * 16 / eo;  // 16-byte row pitch for the TMA store
    p->tmp_bytes = (size_t)M * (size_t)p->tmp_ld * (size_t)eo;
    if (cudaMalloc(&p->d_tmp, p->tmp_bytes) != cudaSuccess) {
      cudaFree(p->d_err);
      delete p;
      return fail(FL_ERR_OOM, "fl_plan: cudaMalloc(unfused intermediate, %zu bytes)", p->tmp_bytes);
    }
  }
  *out = p;
  return FL_OK;
}

// The configuration fl_plan would choose on a device with `num_sms` SMs and
// `max_smem_per_block` bytes of opt-in shared memory per block, without touching any
// device: the same checks, the same choice, nothing allocated.
extern "C" fl_status fl_plan_preview(int64_t M, int64_t N, int64_t K, int32_t dtype, int32_t compute,
                                     const fl_epilogue_desc* epi, int32_t num_sms, int32_t max_smem_per_block,
                                     fl_plan_info* info) {
  g_err[0] = 0;
  if (!epi || !info) return fail(FL_ERR_INVALID_ARG, "fl_plan_preview: null epilogue descriptor or info");
  if (num_sms < 2 || num_sms > 4096 || max_smem_per_block < 16384)
    return fail(FL_ERR_INVALID_ARG, "fl_plan_preview: implausible device (%d SMs, %d bytes of shared memory)",
                num_sms, max_smem_per_block);
  fl_plan_s* p = nullptr;
  const fl_status st = plan_host_part(&p, M, N, K, dtype, compute, epi);
  if (st != FL_OK) return st;
  p->num_sms = num_sms;
  p->max_smem = max_smem_per_block;
  choose_config(p);
  const int b_boxes = b_boxes_of(p, p->epi.kind == FL_EPI_GEGLU_TANH);
  const Layout L = layout_for(p, p->mma_n, b_boxes, p->max_smem);
  fl_status r = FL_OK;
  if (L.stages < 2) {
    r = fail(FL_ERR_UNSUPPORTED, "fl_plan_preview: shared memory too small");
  } else {
    p->stages = L.stages;
    p->smem = (int)L.total;
    p->grid = grid_of(p);
    if (!kernel_of(p, p->act, p->epi.out_dtype)) {
      r = fail(FL_ERR_UNSUPPORTED, "fl_plan_preview: no kernel for this combination");
    } else {
      p->launches = p->epi.unfused ? unfused_launches(p) : 1;
      r = fl_get_plan_info(p, info);
    }
  }
  delete p;
  return r;
}

extern "C" fl_status fl_get_plan_info(fl_plan_t p, fl_plan_info* info) {
  if (!p || !info) return fail(FL_ERR_INVALID_ARG, "fl_get_plan_info: null argument");
  memset(info, 0, sizeof(*info));
  info->tile_m = p->swap ? p->mma_n : (p->pair ? 256 : 128);
  info->tile_n = p->swap ? 128 : p->out_tile_n;
  info->mma_n = p->mma_n;
  info->swap_ab = p->swap ? 1 : 0;
  info->split_k = p->split_k;
  info->stages = p->stages;
  info->grid = p->grid;
  info->smem_bytes = p->smem;
  info->launches_per_execute = p->launches;
  info->cta_pair = p->pair ? 1 : 0;
  info->stream_k_tiles = p->sk_tiles;
  info->stream_k_pairs = p->sk_clusters;
  return FL_OK;
}

extern "C" fl_status fl_free(fl_plan_t p) {
  if (!p) return FL_OK;
  if (p->d_err) cudaFree(p->d_err);
  if (p->d_tmp) cudaFree(p->d_tmp);
  if (p->d_skws) cudaFree(p->d_skws);
  if (p->d_skflags) cudaFree(p->d_skflags);
  delete p;
  return FL_OK;
}

static bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// ------------------------------------------------------------------ launch helpers
struct GemmArgs {
  const void* A;
  const void* W;
  void* out;
  int out_dtype;
  int64_t ldo;
  int act;
  const void* bias;
  const void* residual;
  uint32_t* aux;
  float scale;
  int64_t n_cols;  // columns of the GEMM result written to `out` (N, or 2N for the unfused dual GEMM)
  bool geglu_fused;
};

// Launch an elementwise kernel with programmatic dependent launch allowed.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl_b(void (*kern)(KArgs...), dim3 grid, unsigned block, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(block, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, cudaStream_t s, Args... args) {
  return launch_pdl_b(kern, grid, 256u, s, args...);
}

static fl_status launch_kernel(const fl_plan_s* p, const LaunchCache& c, cudaStream_t stream,
                               const void* kernel, bool swap) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)p->grid, 1, 1);
  cfg.blockDim = dim3(swap ? Cfg<true>::kThreads : Cfg<false>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)p->smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  // programmatic dependent launch: the kernel's prologue may overlap the tail of
  // the previous kernel of the stream (the kernel waits before touching memory)
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (p->split_k > 1 || p->pair) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = p->pair ? 2u : (unsigned)p->split_k;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  cudaError_t err = cudaLaunchKernelEx(&cfg, reinterpret_cast<KernelFn>(const_cast<void*>(kernel)), c.tmA, c.tmB,
                                       c.tmB2, c.tmOut, c.k);
  if (err != cudaSuccess) return fail(FL_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(err));
  return after_launch(stream, "fused GEMM kernel");
}

static fl_status launch_gemm(fl_plan_s* p, const GemmArgs& g, cudaStream_t stream, const void* kernel,
                             bool swap, int act, LaunchCache* cache) {
  const void* key[8] = {g.A, g.W, g.out, g.bias, g.residual, g.aux, kernel, (const void*)(intptr_t)g.ldo};
  if (cache->valid && memcmp(cache->key, key, sizeof(key)) == 0) return launch_kernel(p, *cache, stream, kernel, swap);
  const int es = esize(p->dtype);
  const int bk = p->k_atoms * 128 / es;
  const fl_epilogue_desc& e = p->epi;
  KParams k{};
  k.M = (int)p->M;
  k.N = (int)g.n_cols;
  k.K = (int)p->K;
  k.num_kb = p->num_kb;
  k.split_k = p->split_k;
  k.mma_n = p->mma_n;
  k.out_tile_n = p->out_tile_n;
  k.tiles_a = p->tiles_a;
  k.tiles_b = p->tiles_b;
  k.bk = bk;
  k.b_mn_major = e.b_major;
  k.geglu = g.geglu_fused ? 1 : 0;
  const int b_boxes = b_boxes_of(p, g.geglu_fused);
  Layout L = layout_for(p, p->mma_n, b_boxes, p->max_smem);
  k.num_stages = p->stages;
  k.b_boxes = b_boxes;
  k.b_box_rows = e.b_major ? 64 : (p->pair ? p->mma_n / 2 : p->mma_n) / b_boxes;
  k.a_stage_bytes = L.a_stage;
  k.b_box_bytes = L.b_box;
  k.stage_bytes = L.stage;
  k.stage_stride = L.stride;
  k.k_atoms = p->k_atoms;
  k.a_atom_bytes = 128u * 128u;
  k.b_atom_bytes = e.b_major ? 0u : (uint32_t)(p->pair ? p->mma_n / 2 : p->mma_n) * 128u;
  k.usteps = kUmmaSteps * p->k_atoms;
  k.staging_off = L.staging_off;
  k.bias_off = L.bias_off;
  k.red_off = L.red_off;
  k.red_pitch = L.red_pitch;
  k.res_off = L.res_off;
  k.res_blk_bytes = L.res_blk;
  k.bar_off = L.bar_off;
  const uint32_t fmt = (p->dtype == FL_BF16) ? 1u : (p->dtype == FL_F32 ? 2u : 0u);  // F16 / BF16 / TF32
  k.idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(e.b_major ? 1 : 0) << 16) |
            ((uint32_t)(p->mma_n >> 3) << 17) | ((uint32_t)((p->pair ? 256 : 128) >> 4) << 24);
  k.a_kstep = 32;
  k.b_kstep = e.b_major ? 16u * 128u : 32u;
  k.b_lbo = e.b_major ? L.b_box : 16u;
  int tc = 2 * p->mma_n;
  uint32_t cols = 32;
  while ((int)cols < tc) cols <<= 1;
  k.tmem_cols = cols;
  k.bias = g.bias;
  k.bias_dtype = e.bias_dtype;
  k.bias_axis = e.bias_axis;
  k.residual = g.residual;
  k.ldr = e.ldr;
  k.res_dtype = e.residual_dtype;
  k.res_async = g.residual != nullptr && (reinterpret_cast<uintptr_t>(g.residual) & 15u) == 0;
  k.out = g.out;
  k.ldo = g.ldo;
  k.aux = g.aux;
  k.ld_aux = cdiv(p->M > 0 ? g.n_cols : 0, 32);
  k.scale = g.scale;
  k.err = p->d_err;
  k.wait_limit_ns = p->wait_limit_ns;
  k.sk_tiles = p->sk_tiles;
  k.sk_clusters = p->sk_clusters;
  set_dp_split(k, p->grid / (p->pair ? 2 : std::max(1, p->split_k)));
  k.sk_ws = p->d_skws;
  k.sk_flags = p->d_skflags;

  CUtensorMap tmA, tmB, tmB2, tmOut;
  const int ae = 128 / es;  // K elements of one 128-byte swizzle atom: the inner box of K-major maps
  memset(&tmB2, 0, sizeof(tmB2));
  memset(&tmOut, 0, sizeof(tmOut));
  fl_status st;
  const uint64_t Kd = (uint64_t)std::max<int64_t>(p->K, 1);
  const bool no_k = p->K == 0;  // no operand is read: y = epi(0 + bias)
  memset(&tmA, 0, sizeof(tmA));
  memset(&tmB, 0, sizeof(tmB));
  if (!swap) {
    if (!no_k) st = make_map(&tmA, g.A, p->dtype, Kd, (uint64_t)p->M, (uint64_t)e.lda * es, (uint32_t)ae, 128);
    else st = FL_OK;
    if (st) return st;
    if (no_k) {
      st = FL_OK;
    } else if (e.b_major) {
      st = make_map(&tmB, g.W, p->dtype, (uint64_t)g.n_cols, Kd, (uint64_t)e.ldb * es, 64, (uint32_t)bk);
    } else if (g.geglu_fused) {
      st = make_map(&tmB, g.W, p->dtype, Kd, (uint64_t)p->N, (uint64_t)e.ldb * es, (uint32_t)ae, 128);
      if (st) return st;
      const char* up = static_cast<const char*>(g.W) + (size_t)p->N * (size_t)e.ldb * es;
      st = make_map(&tmB2, up, p->dtype, Kd, (uint64_t)p->N, (uint64_t)e.ldb * es, (uint32_t)ae, 128);
    } else {
      st = make_map(&tmB, g.W, p->dtype, Kd, (uint64_t)g.n_cols, (uint64_t)e.ldb * es, (uint32_t)ae,
                    (uint32_t)(p->pair ? p->mma_n / 2 : p->mma_n));
    }
    if (st) return st;
    // The TMA store covers whole 16-byte granules of a row only; the kernel writes
    // the ragged remainder (< 16 bytes per row) with plain stores.
    const int eo = esize(g.out_dtype);
    const int64_t n_tma = (g.n_cols * eo / 16) * 16 / eo;
    k.n_tma = (int)n_tma;
    st = make_map(&tmOut, g.out, g.out_dtype, (uint64_t)std::max<int64_t>(n_tma, 16 / eo), (uint64_t)p->M,
                  (uint64_t)g.ldo * eo, (uint32_t)(128 / eo), 32);
    if (st) return st;
  } else if (!no_k) {
    // UMMA A = weight rows (output features), UMMA B = activation rows
    st = make_map(&tmA, g.W, p->dtype, Kd, (uint64_t)g.n_cols, (uint64_t)e.ldb * es, (uint32_t)ae, 128);
    if (st) return st;
    st = make_map(&tmB, g.A, p->dtype, Kd, (uint64_t)p->M, (uint64_t)e.lda * es, (uint32_t)ae,
                  (uint32_t)p->mma_n);
    if (st) return st;
    tmOut = tmA;  // unused in the swap layout
  } else {
    tmOut = tmA;  // unused in the swap layout
  }
  if (!g.geglu_fused) tmB2 = tmB;  // unused
  (void)act;
  cache->tmA = tmA;
  cache->tmB = tmB;
  cache->tmB2 = tmB2;
  cache->tmOut = tmOut;
  cache->k = k;
  memcpy(cache->key, key, sizeof(key));
  cache->valid = true;
  return launch_kernel(p, *cache, stream, kernel, swap);
}

static int grid_for(long long work, int num_sms) {
  long long b = (work + 255) / 256;
  long long cap = (long long)num_sms * 8;
  if (b > cap) b = cap;
  if (b < 1) b = 1;
  return (int)b;
}

// One wave of resident 256-thread CTAs for a grid-stride kernel whose warps take `units`
// work units in turn.  A grid larger than one wave leaves a partial second wave of CTAs; a
// grid of exactly one wave can leave some warps a unit more than the rest.  So: the fewest
// rounds of units one wave needs, then the fewest warps that finish in that many rounds.
static int resident_grid(const void* kernel, long long units, int num_sms) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, 0) != cudaSuccess || per_sm < 1) {
    (void)cudaGetLastError();
    per_sm = 1;
  }
  const long long slots = (long long)num_sms * per_sm * 8;
  const long long rounds = std::max<long long>(1, (units + slots - 1) / slots);
  const long long warps = (units + rounds - 1) / rounds;
  return (int)std::max<long long>(1, (warps + 7) / 8);
}

template <int DT>
static fl_status launch_ew_t(const EwParams& P, int num_sms, cudaStream_t s) {
  constexpr int es = (DT == DT_F32) ? 4 : 2;
  const bool vec = aligned16(P.src) && aligned16(P.dst) && (P.lds * es) % 16 == 0 && (P.ldd * es) % 16 == 0;
  cudaError_t err;
  if (vec) {
    // one thread per 16-byte vector slot (rows padded to whole mask words)
    const long long work = P.M * ((P.N + 31) / 32) * (32 / (16 / es));
    err = launch_pdl(fl_ew_step_vec_kernel<DT>, dim3((unsigned)grid_for(work, num_sms)), s, P);
  } else {
    const long long work = P.M * ((P.N + 31) / 32);
    err = launch_pdl(fl_ew_step_kernel<DT>, dim3((unsigned)grid_for(work, num_sms)), s, P);
  }
  if (err != cudaSuccess) return fail(FL_ERR_CUDA, "elementwise kernel launch: %s", cudaGetErrorString(err));
  return after_launch(s, "elementwise step kernel");
}
static fl_status launch_ew(int dt, const EwParams& P, int num_sms, cudaStream_t s) {
  if (dt == FL_BF16) return launch_ew_t<DT_BF16>(P, num_sms, s);
  if (dt == FL_F16) return launch_ew_t<DT_F16>(P, num_sms, s);
  return launch_ew_t<DT_F32>(P, num_sms, s);
}

// ------------------------------------------------------------------ execute
extern "C" fl_status fl_execute(fl_plan_t p, const void* A, const void* W, const void* bias, void* aux_,
                                const void* residual, void* out, void* stream_) {
  g_err[0] = 0;
  uint32_t* aux = static_cast<uint32_t*>(aux_);
  if (!p) return fail(FL_ERR_INVALID_ARG, "fl_execute: null plan");
  if (!out || (p->K > 0 && (!A || !W)))
    return fail(FL_ERR_INVALID_ARG, "fl_execute: A, W (when K > 0) and out are required");
  if (p->has_bias && !bias) return fail(FL_ERR_INVALID_ARG, "fl_execute: this epilogue needs a bias");
  if (!p->has_bias && bias) return fail(FL_ERR_INVALID_ARG, "fl_execute: this epilogue takes no bias");
  if (p->has_aux && !aux) return fail(FL_ERR_INVALID_ARG, "fl_execute: RELU_AUX_BIAS / GELU_AUX_BIAS need the aux buffer");
  if (!p->has_aux && aux) return fail(FL_ERR_INVALID_ARG, "fl_execute: only the AUX epilogues write an aux buffer");
  if (aux && p->epi.kind == FL_EPI_GELU_AUX_BIAS && !aligned16(aux))
    return fail(FL_ERR_ALIGNMENT, "fl_execute: the GELU_AUX_BIAS pre-activation buffer must be 16-byte aligned");
  if (p->epi.has_residual && !residual) return fail(FL_ERR_INVALID_ARG, "fl_execute: has_residual needs a residual");
  if (!p->epi.has_residual && residual) return fail(FL_ERR_INVALID_ARG, "fl_execute: residual given but not planned");
  if ((p->K > 0 && (!aligned16(A) || !aligned16(W))) || !aligned16(out) || (residual && !aligned16(residual)))
    return fail(FL_ERR_ALIGNMENT, "fl_execute: A, W, out and residual must be 16-byte aligned");
  if (bias && (reinterpret_cast<uintptr_t>(bias) % (uintptr_t)esize(p->epi.bias_dtype)))
    return fail(FL_ERR_ALIGNMENT, "fl_execute: bias is not aligned to its element size");
  if (aux && (reinterpret_cast<uintptr_t>(aux) & 3u)) return fail(FL_ERR_ALIGNMENT, "fl_execute: aux must be 4-byte aligned");
  int dev = -1;
  FL_CUDA(cudaGetDevice(&dev));
  if (dev != p->device) return fail(FL_ERR_INVALID_ARG, "fl_execute: plan was made on device %d, current is %d", p->device, dev);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const fl_epilogue_desc& e = p->epi;
  const bool geglu = e.kind == FL_EPI_GEGLU_TANH;

  if (!e.unfused) {
    GemmArgs g{A, W, out, e.out_dtype, e.ldo, p->act, bias, residual, aux, e.scale, p->N, geglu};
    return launch_gemm(p, g, stream, p->kernel, p->swap, p->act, &p->cache_fused);
  }

  // ---- unfused twin: bare GEMM into the intermediate, then one kernel per step
  const int odt = e.out_dtype;
  const int64_t cols = geglu ? 2 * p->N : p->N;
  const bool no_steps = (e.kind == FL_EPI_NONE) && !e.has_residual && e.scale == 1.0f;
  void* gemm_out = no_steps ? out : p->d_tmp;
  const int64_t gemm_ld = no_steps ? e.ldo : p->tmp_ld;
  {
    // The unfused GEMM uses the same tcgen05 kernel with no epilogue work.
    fl_plan_s q;
    twin_config(p, &q);
    const void* kern = kernel_of(&q, ACT_NONE, odt);
    q.epi.ldr = 0;
    q.epi.has_residual = 0;
    GemmArgs g{A, W, gemm_out, odt, gemm_ld, ACT_NONE, nullptr, nullptr, nullptr, 1.0f, cols, false};
    fl_status st = launch_gemm(&q, g, stream, kern, q.swap, ACT_NONE, &p->cache_unfused);
    if (st) return st;
  }
  if (no_steps) return FL_OK;
  EwParams P{};
  P.M = p->M;
  P.N = p->N;
  P.src = p->d_tmp;
  P.lds = p->tmp_ld;
  P.dst = out;
  P.ldd = e.ldo;
  P.err = p->d_err;
  const long long tmp_elems = (long long)(p->tmp_bytes / (size_t)esize(odt));
  const long long out_elems = (p->M - 1) * e.ldo + p->N;
  P.src_elems = tmp_elems;
  P.dst_elems = out_elems;
  P.aux_elems = p->M * cdiv(p->N, 32);
  auto step = [&](int op, const void* operand, int odtype, int64_t ldop) -> fl_status {
    P.op = op;
    P.operand = operand;
    P.operand_dtype = odtype;
    P.ldop = ldop;
    if (op == EW_BIAS_N) P.op_elems = p->N;
    else if (op == EW_BIAS_M) P.op_elems = p->M;
    else if (op == EW_RESIDUAL) P.op_elems = (p->M - 1) * e.ldr + p->N;
    else if (op == EW_GEGLU_MUL) P.op_elems = tmp_elems - p->N;
    else P.op_elems = 0;
    fl_status st = launch_ew(odt, P, p->num_sms, stream);
    P.src = out;  // every later step works in place on `out`
    P.lds = e.ldo;
    P.src_elems = out_elems;
    return st;
  };
  fl_status st = FL_OK;
  if (geglu) {
    // h = gelu_tanh(g) * u, with g = tmp[:, :N] and u = tmp[:, N:]
    P.op = EW_GEGLU_MUL;
    st = step(EW_GEGLU_MUL, static_cast<const char*>(p->d_tmp) + (size_t)p->N * esize(odt), odt, p->tmp_ld);
    if (st) return st;
  } else {
    if (p->has_bias) {
      st = step(e.bias_axis == 0 ? EW_BIAS_N : EW_BIAS_M, bias, e.bias_dtype, 0);
      if (st) return st;
    }
    if (p->act == ACT_RELU) {
      P.aux = aux;
      P.ld_aux = cdiv(p->N, 32);
      st = step(EW_RELU, nullptr, 0, 0);
      P.aux = nullptr;
    } else if (p->act == ACT_GELU) {
      st = step(EW_GELU, nullptr, 0, 0);
    } else if (p->act == ACT_GELU_TANH) {
      st = step(EW_GELU_TANH, nullptr, 0, 0);
    } else if (p->act == ACT_GELU_SIGMOID) {
      st = step(EW_GELU_SIGMOID, nullptr, 0, 0);
    }
    if (st) return st;
  }
  if (e.has_residual) {
    st = step(EW_RESIDUAL, residual, e.residual_dtype, e.ldr);
    if (st) return st;
  }
  if (e.scale != 1.0f) {
    P.scale = e.scale;
    st = step(EW_SCALE, nullptr, 0, 0);
    if (st) return st;
  }
  if (P.src == p->d_tmp) {  // no step ran (e.g. NONE with nothing else): copy through
    FL_CUDA(cudaMemcpy2DAsync(out, (size_t)e.ldo * esize(odt), p->d_tmp, (size_t)p->tmp_ld * esize(odt),
                              (size_t)p->N * esize(odt), (size_t)p->M, cudaMemcpyDeviceToDevice, stream));
  }
  return FL_OK;
}

// ------------------------------------------------------------------ dReLU
extern "C" fl_status fl_relu_backward(const void* grad, const uint32_t* aux, void* dpre, int64_t M, int64_t N,
                                      int64_t ld_grad, int64_t ld_dpre, int32_t dtype, void* stream_) {
  g_err[0] = 0;
  if (!grad || !aux || !dpre) return fail(FL_ERR_INVALID_ARG, "fl_relu_backward: null pointer");
  if (M < 0 || N < 0) return fail(FL_ERR_INVALID_ARG, "fl_relu_backward: negative size");
  if (dtype != FL_F16 && dtype != FL_BF16 && dtype != FL_F32)
    return fail(FL_ERR_INVALID_ARG, "fl_relu_backward: unknown dtype %d", dtype);
  if (ld_grad == 0) ld_grad = N;
  if (ld_dpre == 0) ld_dpre = N;
  if (ld_grad < N || ld_dpre < N) return fail(FL_ERR_INVALID_ARG, "fl_relu_backward: leading dimension < N");
  const int es = esize(dtype);
  if (reinterpret_cast<uintptr_t>(grad) % es || reinterpret_cast<uintptr_t>(dpre) % es ||
      reinterpret_cast<uintptr_t>(aux) % 4)
    return fail(FL_ERR_ALIGNMENT, "fl_relu_backward: misaligned pointer");
  if (M == 0 || N == 0) return FL_OK;
  const int vec_ok = aligned16(grad) && aligned16(dpre) && (ld_grad * es) % 16 == 0 && (ld_dpre * es) % 16 == 0;
  int dev = 0, sms = 148;
  FL_CUDA(cudaGetDevice(&dev));
  FL_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const long long words = cdiv(N, 32);
  const long long units = M * cdiv(words, 32);  // a warp takes 32 mask words of a row per round
  const void* kern = dtype == FL_BF16 ? (const void*)fl_relu_backward_kernel<DT_BF16>
                   : dtype == FL_F16  ? (const void*)fl_relu_backward_kernel<DT_F16>
                                      : (const void*)fl_relu_backward_kernel<DT_F32>;
  const int grid = resident_grid(kern, units, sms);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
  cudaError_t err;
  if (dtype == FL_BF16)
    err = launch_pdl(fl_relu_backward_kernel<DT_BF16>, dim3((unsigned)grid), s, grad, aux, dpre, (long long)M, (long long)N,
                     (long long)ld_grad, (long long)ld_dpre, words, vec_ok);
  else if (dtype == FL_F16)
    err = launch_pdl(fl_relu_backward_kernel<DT_F16>, dim3((unsigned)grid), s, grad, aux, dpre, (long long)M, (long long)N,
                     (long long)ld_grad, (long long)ld_dpre, words, vec_ok);
  else
    err = launch_pdl(fl_relu_backward_kernel<DT_F32>, dim3((unsigned)grid), s, grad, aux, dpre, (long long)M, (long long)N,
                     (long long)ld_grad, (long long)ld_dpre, words, vec_ok);
  if (err != cudaSuccess) return fail(FL_ERR_CUDA, "dReLU kernel launch: %s", cudaGetErrorString(err));
  return after_launch(s, "dReLU kernel");
}

// ------------------------------------------------------------------ backward with bias gradient
// Launch geometry of fl_bwd_bgrad_kernel: column groups of eight strips of 32 16-byte
// vectors, and row blocks enough for one resident wave of three CTAs per SM; the
// workspace holds one row of fp32 column partial sums per row block.
struct BwdGeom {
  int groups, row_blocks, rows_per_block;
  long long ws_ld;
  size_t bytes;
};
static fl_status bwd_geom(int64_t M, int64_t N, int dtype, BwdGeom* g) {
  int dev = 0, sms = 148;
  FL_CUDA(cudaGetDevice(&dev));
  FL_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const int ve = 16 / esize(dtype);
  g->groups = (int)std::max<int64_t>(1, cdiv(N, 8LL * 32LL * ve));
  int64_t rb = std::max<int64_t>(1, cdiv(3LL * sms, g->groups));
  rb = std::min<int64_t>(rb, std::max<int64_t>(1, M));
  g->rows_per_block = (int)std::max<int64_t>(1, cdiv(M, rb));
  g->row_blocks = (int)std::max<int64_t>(1, cdiv(M, g->rows_per_block));
  g->ws_ld = (long long)g->groups * 8LL * 32LL * ve;
  g->bytes = (size_t)g->row_blocks * (size_t)g->ws_ld * sizeof(float);
  return FL_OK;
}

extern "C" fl_status fl_bias_grad_workspace_size(int64_t M, int64_t N, int32_t dtype, size_t* bytes) {
  g_err[0] = 0;
  if (!bytes) return fail(FL_ERR_INVALID_ARG, "fl_bias_grad_workspace_size: null pointer");
  if (M < 0 || N < 0) return fail(FL_ERR_INVALID_ARG, "fl_bias_grad_workspace_size: negative size");
  if (dtype != FL_F16 && dtype != FL_BF16 && dtype != FL_F32)
    return fail(FL_ERR_INVALID_ARG, "fl_bias_grad_workspace_size: unknown dtype %d", dtype);
  BwdGeom g;
  fl_status st = bwd_geom(M, N, dtype, &g);
  if (st) return st;
  *bytes = g.bytes;
  return FL_OK;
}

static fl_status bwd_bgrad(int mode, const char* who, const void* grad, const uint32_t* mask, const void* v, void* dpre,
                           float* dbias, int64_t M, int64_t N, int64_t ld_grad, int64_t ld_v, int64_t ld_dpre,
                           int32_t dtype, void* workspace, size_t workspace_bytes, void* stream_) {
  g_err[0] = 0;
  if (!grad || !dpre || (mode == BWD_DRELU ? !mask : !v)) return fail(FL_ERR_INVALID_ARG, "%s: null pointer", who);
  if (M < 0 || N < 0) return fail(FL_ERR_INVALID_ARG, "%s: negative size", who);
  if (dtype != FL_F16 && dtype != FL_BF16 && dtype != FL_F32)
    return fail(FL_ERR_INVALID_ARG, "%s: unknown dtype %d", who, dtype);
  if (ld_grad == 0) ld_grad = N;
  if (ld_dpre == 0) ld_dpre = N;
  if (ld_v == 0) ld_v = N;
  if (ld_grad < N || ld_dpre < N || (mode == BWD_DGELU && ld_v < N))
    return fail(FL_ERR_INVALID_ARG, "%s: leading dimension < N", who);
  const int es = esize(dtype);
  if (reinterpret_cast<uintptr_t>(grad) % es || reinterpret_cast<uintptr_t>(dpre) % es ||
      (mask && reinterpret_cast<uintptr_t>(mask) % 4) || (v && reinterpret_cast<uintptr_t>(v) % es) ||
      (dbias && reinterpret_cast<uintptr_t>(dbias) % 4))
    return fail(FL_ERR_ALIGNMENT, "%s: misaligned pointer", who);
  BwdGeom g;
  fl_status st = bwd_geom(M, N, dtype, &g);
  if (st) return st;
  if (dbias && (!workspace || workspace_bytes < g.bytes || !aligned16(workspace)))
    return fail(FL_ERR_INVALID_ARG, "%s: the bias gradient needs a 16-byte aligned workspace of "
                "%zu bytes (fl_bias_grad_workspace_size)", who, g.bytes);
  if (M == 0 || N == 0) {
    if (dbias && N > 0) FL_CUDA(cudaMemsetAsync(dbias, 0, (size_t)N * sizeof(float), (cudaStream_t)stream_));
    return FL_OK;
  }
  BwdParams P{};
  P.grad = grad;
  P.mask = mask;
  P.v = v;
  P.dpre = dpre;
  P.dbias = dbias;
  P.ws = dbias ? reinterpret_cast<float*>(workspace) : nullptr;
  P.M = M;
  P.N = N;
  P.ldg = ld_grad;
  P.ldv = ld_v;
  P.ldd = ld_dpre;
  P.words = cdiv(N, 32);
  P.ws_ld = g.ws_ld;
  P.rows_per_block = g.rows_per_block;
  P.row_blocks = g.row_blocks;
  P.vec_ok = aligned16(grad) && aligned16(dpre) && (ld_grad * es) % 16 == 0 && (ld_dpre * es) % 16 == 0 &&
             (mode == BWD_DRELU || (aligned16(v) && (ld_v * es) % 16 == 0));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
  const dim3 grid((unsigned)g.groups, (unsigned)g.row_blocks);
  cudaError_t err;
  if (mode == BWD_DRELU) {
    err = dtype == FL_BF16 ? launch_pdl(fl_bwd_bgrad_kernel<DT_BF16, BWD_DRELU>, grid, s, P)
        : dtype == FL_F16  ? launch_pdl(fl_bwd_bgrad_kernel<DT_F16, BWD_DRELU>, grid, s, P)
                           : launch_pdl(fl_bwd_bgrad_kernel<DT_F32, BWD_DRELU>, grid, s, P);
  } else {
    err = dtype == FL_BF16 ? launch_pdl(fl_bwd_bgrad_kernel<DT_BF16, BWD_DGELU>, grid, s, P)
        : dtype == FL_F16  ? launch_pdl(fl_bwd_bgrad_kernel<DT_F16, BWD_DGELU>, grid, s, P)
                           : launch_pdl(fl_bwd_bgrad_kernel<DT_F32, BWD_DGELU>, grid, s, P);
  }
  if (err != cudaSuccess) return fail(FL_ERR_CUDA, "%s: kernel launch: %s", who, cudaGetErrorString(err));
  if (dbias) {
    // the column sums of the row blocks' partials, in a fixed order
    err = launch_pdl_b(fl_bgrad_reduce_kernel, dim3((unsigned)cdiv(N, 32)), 1024u, s, (const float*)P.ws, dbias,
                       (long long)N, (long long)g.ws_ld, g.row_blocks);
    if (err != cudaSuccess) return fail(FL_ERR_CUDA, "%s: reduction kernel launch: %s", who, cudaGetErrorString(err));
  }
  return after_launch(s, who);
}

extern "C" fl_status fl_drelu_bgrad(const void* grad, const uint32_t* aux, void* dpre, float* dbias, int64_t M,
                                    int64_t N, int64_t ld_grad, int64_t ld_dpre, int32_t dtype, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  return bwd_bgrad(BWD_DRELU, "fl_drelu_bgrad", grad, aux, nullptr, dpre, dbias, M, N, ld_grad, 0, ld_dpre, dtype,
                   workspace, workspace_bytes, stream);
}

extern "C" fl_status fl_dgelu_bgrad(const void* grad, const void* v, void* dpre, float* dbias, int64_t M, int64_t N,
                                    int64_t ld_grad, int64_t ld_v, int64_t ld_dpre, int32_t dtype, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  return bwd_bgrad(BWD_DGELU, "fl_dgelu_bgrad", grad, nullptr, v, dpre, dbias, M, N, ld_grad, ld_v, ld_dpre, dtype,
                   workspace, workspace_bytes, stream);
}

// ------------------------------------------------------------------ failure-path self-test
extern "C" fl_status fl_wait_selftest(uint64_t limit_ns, void* stream_) {
  g_err[0] = 0;
  if (limit_ns == 0 || limit_ns > 10000000000ull)
    return fail(FL_ERR_INVALID_ARG, "fl_wait_selftest: limit must be in (0, 10 s]");
  int* d_err = nullptr;
  FL_CUDA(cudaMalloc(&d_err, sizeof(int)));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
  fl_status st = FL_OK;
  if (cudaMemsetAsync(d_err, 0, sizeof(int), s) != cudaSuccess) st = fail(FL_ERR_CUDA, "fl_wait_selftest: memset");
  if (!st) {
    fl_wait_selftest_kernel<<<1, 32, 0, s>>>(d_err, (unsigned long long)limit_ns);
    st = after_launch(s, "fl_wait_selftest");
  }
  int h = 0;
  if (!st && cudaStreamSynchronize(s) != cudaSuccess) st = fail(FL_ERR_CUDA, "fl_wait_selftest: synchronize");
  if (!st && cudaMemcpy(&h, d_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    st = fail(FL_ERR_CUDA, "fl_wait_selftest: read back");
  cudaFree(d_err);
  if (st) return st;
  // the wait must have given up: the bounded-wait failure path reports a timeout
  if (h == 0) return fail(FL_ERR_CUDA, "fl_wait_selftest: the wait did not report its timeout");
  return fail(FL_ERR_TIMEOUT, "fl_wait_selftest: the bounded wait gave up as designed (code %d)", h);
}

// ------------------------------------------------------------------ LayerNorm after the tail
template <int XT, int ZT, int TPB>
static void (*ln_kernel(bool vec))(LnParams) {
  return vec ? fl_layernorm_vec_kernel<XT, ZT, TPB> : fl_layernorm_kernel<XT, ZT, TPB>;
}

// The kernel loops over rows: the grid is one resident wave, or M CTAs if fewer.
template <int XT, int TPB>
static cudaError_t launch_ln_w(int z_dtype, cudaStream_t s, const LnParams& P) {
  int dev = 0, sms = 148, per_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // whole-vector layout: every access of the row, the parameters and z is a 16-byte vector
  constexpr long long ve = 16 / (XT == DT_F32 ? 4 : 2);
  constexpr long long vmax = TPB == 128 ? 32 / ve : 4;
  const bool vec = P.vec_ok && P.pvec && P.zvec && P.N % ve == 0 && P.N <= TPB * vmax * ve;
  void (*k)(LnParams) = z_dtype == FL_BF16 ? ln_kernel<XT, DT_BF16, TPB>(vec)
                      : z_dtype == FL_F16  ? ln_kernel<XT, DT_F16, TPB>(vec)
                                           : ln_kernel<XT, DT_F32, TPB>(vec);
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, (const void*)k, TPB, 0);
  if (e != cudaSuccess) return e;
  const long long wave = (long long)std::max(1, per_sm) * sms;
  return launch_pdl_b(k, dim3((unsigned)std::min<long long>(P.M, wave)), TPB, s, P);
}

// Rows of up to 8 KB take 128 threads (32 elements a thread); longer rows 256, four CTAs
// per SM (on 2048 x 4096 fp32 rows, 256 threads measured 11.2 us against 13.3 us for 128,
// and four 256-thread CTAs per SM 11.1-11.4 against 11.4-11.8 for three).
template <int XT>
static cudaError_t launch_ln(int z_dtype, cudaStream_t s, const LnParams& P) {
  const long long row_bytes = P.N * (XT == DT_F32 ? 4 : 2);
  if (P.N <= 128 * 32 && row_bytes <= 8192) return launch_ln_w<XT, 128>(z_dtype, s, P);
  return launch_ln_w<XT, 256>(z_dtype, s, P);
}

extern "C" fl_status fl_layernorm(const void* x, const void* gamma, const void* beta, void* z, int64_t M, int64_t N,
                                  int64_t ld_x, int64_t ld_z, int32_t x_dtype, int32_t z_dtype, int32_t param_dtype,
                                  float eps, void* stream_) {
  g_err[0] = 0;
  const char* who = "fl_layernorm";
  if (!x || !z) return fail(FL_ERR_INVALID_ARG, "%s: null x or z", who);
  if (M < 0 || N < 0) return fail(FL_ERR_INVALID_ARG, "%s: negative size", who);
  for (int dt : {x_dtype, z_dtype, param_dtype})
    if (dt != FL_F16 && dt != FL_BF16 && dt != FL_F32) return fail(FL_ERR_INVALID_ARG, "%s: unknown dtype %d", who, dt);
  if (!(eps >= 0.0f)) return fail(FL_ERR_INVALID_ARG, "%s: eps must be >= 0", who);
  if (M > 0x7fffffffLL) return fail(FL_ERR_INVALID_ARG, "%s: more than 2^31-1 rows", who);
  if (ld_x == 0) ld_x = N;
  if (ld_z == 0) ld_z = N;
  if (ld_x < N || ld_z < N) return fail(FL_ERR_INVALID_ARG, "%s: leading dimension < N", who);
  const int ex = esize(x_dtype), ez = esize(z_dtype), ep = esize(param_dtype);
  if (reinterpret_cast<uintptr_t>(x) % ex || reinterpret_cast<uintptr_t>(z) % ez ||
      (gamma && reinterpret_cast<uintptr_t>(gamma) % ep) || (beta && reinterpret_cast<uintptr_t>(beta) % ep))
    return fail(FL_ERR_ALIGNMENT, "%s: misaligned pointer", who);
  if (M == 0 || N == 0) return FL_OK;
  LnParams P{};
  P.x = x;
  P.gamma = gamma;
  P.beta = beta;
  P.z = z;
  P.M = M;
  P.N = N;
  P.ldx = ld_x;
  P.ldz = ld_z;
  P.param_dtype = param_dtype;
  P.vec_ok = aligned16(x) && (ld_x * ex) % 16 == 0;
  P.pvec = (!gamma || aligned16(gamma)) && (!beta || aligned16(beta));
  // a thread's VE outputs (VE = 16 bytes of x) start on a multiple of their own size
  P.zvec = aligned16(z) && (ld_z * ez) % 16 == 0 && P.vec_ok;
  P.eps = eps;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
  cudaError_t err = x_dtype == FL_BF16 ? launch_ln<DT_BF16>(z_dtype, s, P)
                    : x_dtype == FL_F16 ? launch_ln<DT_F16>(z_dtype, s, P)
                                        : launch_ln<DT_F32>(z_dtype, s, P);
  if (err != cudaSuccess) return fail(FL_ERR_CUDA, "%s: kernel launch: %s", who, cudaGetErrorString(err));
  return after_launch(s, who);
}

// ------------------------------------------------------------------ status
extern "C" fl_status fl_check_status(fl_plan_t p, void* stream_) {
  if (!p) return fail(FL_ERR_INVALID_ARG, "fl_check_status: null plan");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
  FL_CUDA(cudaStreamSynchronize(s));
  int h = 0;
  FL_CUDA(cudaMemcpy(&h, p->d_err, sizeof(int), cudaMemcpyDeviceToHost));
  if (h != 0) {
    FL_CUDA(cudaMemset(p->d_err, 0, sizeof(int)));
    // a launch that gave up may have left stream-K flags set: clear them for the next one
    if (p->d_skflags) FL_CUDA(cudaMemset(p->d_skflags, 0, p->skflags_bytes));
    if (h >= 100)
      return fail(FL_ERR_DEVICE, "an elementwise kernel skipped an out-of-range access (code %d)", h);
    return fail(FL_ERR_TIMEOUT, "a bounded in-kernel wait gave up (code %d)", h);
  }
  return FL_OK;
}

// ------------------------------------------------------------------ entry point without allocation
// For callers that must not allocate device memory: a host that hands all GPU
// memory to its own pool (an allocation outside it could fragment the pool or
// fail under memory pressure), or a latency-critical path on which cudaMalloc
// and cudaFree are forbidden because they can synchronise the device.  Such a
// caller passes inputs and outputs as usual; the scratch that the planned path
// allocates (the device error word, and the intermediate of the unfused path)
// comes from the fixed array below, which every GPU that loads this library
// holds until the process exits.
static constexpr size_t kNoallocHeadBytes = 256;               // device error word
static constexpr size_t kNoallocTmpBytes = size_t(32) << 20;   // unfused intermediate, at most 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocHeadBytes + kNoallocTmpBytes];

static constexpr int kMaxDevices = 64;
static void* g_noalloc_ptr[kMaxDevices] = {};
static std::mutex g_noalloc_mu;

// Device address of the scratch array on `dev`, looked up once per device with
// that device current (in host code the array's name is only a stand-in).
static fl_status noalloc_scratch(int dev, unsigned char** out) {
  if (dev < 0 || dev >= kMaxDevices) return fail(FL_ERR_DEVICE, "fl_execute_noalloc: device %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return fail(FL_ERR_CUDA, "fl_execute_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = ptr;
  }
  *out = static_cast<unsigned char*>(g_noalloc_ptr[dev]);
  return FL_OK;
}

extern "C" fl_status fl_execute_noalloc(int64_t M, int64_t N, int64_t K, int32_t dtype, int32_t compute,
                                        const fl_epilogue_desc* epi, const void* A, const void* W,
                                        const void* bias, void* aux_, const void* residual, void* out,
                                        void* stream_) {
  g_err[0] = 0;
  uint32_t* aux = static_cast<uint32_t*>(aux_);
  const char* who = "fl_execute_noalloc";
  if (!epi) return fail(FL_ERR_INVALID_ARG, "%s: null epilogue descriptor", who);
  if (M < 1 || N < 1 || K < 0) return fail(FL_ERR_INVALID_ARG, "%s: need M>=1, N>=1, K>=0", who);
  if (M > (1LL << 31) - 256 || N > (1LL << 30) || K > (1LL << 31) - 256)
    return fail(FL_ERR_INVALID_ARG, "%s: dimension too large", who);
  if (epi->kind < FL_EPI_NONE || epi->kind > FL_EPI_GELU_SIGMOID_BIAS)
    return fail(FL_ERR_INVALID_ARG, "%s: unknown epilogue kind %d", who, epi->kind);
  for (int i = 0; i < 2; ++i)
    if (epi->reserved[i] != 0) return fail(FL_ERR_INVALID_ARG, "%s: reserved fields must be 0", who);
  if (epi->schedule < FL_SCHED_AUTO || epi->schedule > FL_SCHED_STREAM_K)
    return fail(FL_ERR_INVALID_ARG, "%s: unknown schedule %d", who, epi->schedule);
  if (dtype != FL_F16 && dtype != FL_BF16) {
    if (dtype == FL_F32) return fail(FL_ERR_UNSUPPORTED, "%s: fp32 operands are not offered", who);
    return fail(FL_ERR_INVALID_ARG, "%s: unknown dtype %d", who, dtype);
  }
  if (compute != FL_COMPUTE_32F) return fail(FL_ERR_UNSUPPORTED, "%s: compute type %d not offered", who, compute);
  if (epi->out_dtype < FL_F16 || epi->out_dtype > FL_F32)
    return fail(FL_ERR_INVALID_ARG, "%s: unknown out_dtype %d", who, epi->out_dtype);
  const bool has_bias = epi->kind != FL_EPI_NONE && epi->kind != FL_EPI_GEGLU_TANH;
  if (has_bias && (epi->bias_dtype < FL_F16 || epi->bias_dtype > FL_F32))
    return fail(FL_ERR_INVALID_ARG, "%s: unknown bias_dtype %d", who, epi->bias_dtype);
  if (epi->has_residual && (epi->residual_dtype < FL_F16 || epi->residual_dtype > FL_F32))
    return fail(FL_ERR_INVALID_ARG, "%s: unknown residual_dtype %d", who, epi->residual_dtype);
  if ((epi->bias_axis != 0 && epi->bias_axis != 1) || (epi->b_major != 0 && epi->b_major != 1))
    return fail(FL_ERR_INVALID_ARG, "%s: bias_axis and b_major must be 0 or 1", who);
  if (epi->kind == FL_EPI_GELU_AUX_BIAS && epi->unfused)
    return fail(FL_ERR_UNSUPPORTED, "%s: the unfused twin has no GELU_AUX_BIAS step", who);
  if (epi->kind == FL_EPI_GEGLU_TANH && (epi->b_major || epi->out_dtype == FL_F32))
    return fail(FL_ERR_UNSUPPORTED, "%s: GEGLU_TANH takes the stacked [2N,K] weight and writes f16/bf16", who);
  if (epi->lda < 0 || epi->ldb < 0 || epi->ldo < 0 || epi->ldr < 0)
    return fail(FL_ERR_INVALID_ARG, "%s: negative leading dimension", who);

  // A plan on the host stack: the same configuration choice as fl_plan, but its
  // scratch points into the fixed array instead of fresh allocations.
  fl_plan_s p{};
  p.M = M; p.N = N; p.K = K; p.dtype = dtype; p.compute = compute; p.epi = *epi;
  p.no_sk = true;  // the stream-K schedule needs a workspace: data-parallel tiles only
  if (p.epi.scale == 0.0f) p.epi.scale = 1.0f;
  p.act = act_of(epi->kind);
  p.has_bias = has_bias;
  p.has_aux = epi->kind == FL_EPI_RELU_AUX_BIAS || epi->kind == FL_EPI_GELU_AUX_BIAS;
  const int64_t a_cols = K, b_cols = epi->b_major ? N : K;
  if (p.epi.lda == 0) p.epi.lda = a_cols;
  if (p.epi.ldb == 0) p.epi.ldb = b_cols;
  if (p.epi.ldo == 0) p.epi.ldo = N;
  if (p.epi.ldr == 0) p.epi.ldr = N;
  if (p.epi.lda < a_cols || p.epi.ldb < b_cols || p.epi.ldo < N || (epi->has_residual && p.epi.ldr < N))
    return fail(FL_ERR_INVALID_ARG, "%s: leading dimension smaller than the row length", who);
  const int es = esize(dtype), eo = esize(epi->out_dtype);
  if ((p.epi.lda * es) % 16 || (p.epi.ldb * es) % 16 || (p.epi.ldo * eo) % 16 ||
      (epi->has_residual && (p.epi.ldr * esize(epi->residual_dtype)) % 16))
    return fail(FL_ERR_ALIGNMENT, "%s: every row pitch must be a multiple of 16 bytes", who);
  if (cudaGetDevice(&p.device) != cudaSuccess) return fail(FL_ERR_DEVICE, "%s: no CUDA device", who);
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, p.device) != cudaSuccess || major != 10)
    return fail(FL_ERR_DEVICE, "%s: needs an sm_100 (B200-class) GPU", who);
  FL_CUDA(cudaDeviceGetAttribute(&p.num_sms, cudaDevAttrMultiProcessorCount, p.device));
  FL_CUDA(cudaDeviceGetAttribute(&p.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, p.device));
  fl_status st = get_encode();
  if (st != FL_OK) return st;

  choose_config(&p);
  const int b_boxes = b_boxes_of(&p, epi->kind == FL_EPI_GEGLU_TANH);
  Layout L = layout_for(&p, p.mma_n, b_boxes, p.max_smem);
  if (L.stages < 2) return fail(FL_ERR_UNSUPPORTED, "%s: shared memory too small", who);
  p.stages = L.stages;
  p.smem = (int)L.total;
  const int tiles = p.tiles_a * p.tiles_b;
  (void)tiles;
  p.grid = grid_of(&p);
  p.kernel = kernel_of(&p, p.act, epi->out_dtype);
  if (!p.kernel) return fail(FL_ERR_UNSUPPORTED, "%s: no kernel for this combination", who);
  FL_CUDA(cudaFuncSetAttribute(p.kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, p.max_smem));
  p.launches = 1;
  p.wait_limit_ns = g_wait_limit_ns;

  unsigned char* scratch = nullptr;
  st = noalloc_scratch(p.device, &scratch);
  if (st != FL_OK) return st;
  p.d_err = reinterpret_cast<int*>(scratch);
  if (epi->unfused) {
    const int64_t cols = (epi->kind == FL_EPI_GEGLU_TANH) ? 2 * N : N;
    p.tmp_ld = cdiv(cols * eo, 16) * 16 / eo;
    const double need = (double)M * (double)p.tmp_ld * (double)eo;
    if (need > (double)kNoallocTmpBytes)
      return fail(FL_ERR_INVALID_ARG, "%s: the unfused intermediate needs %.0f bytes, above the %zu-byte scratch", who,
                  need, kNoallocTmpBytes);
    p.tmp_bytes = (size_t)need;
    p.d_tmp = scratch + kNoallocHeadBytes;
    for (int sw = 0; sw < 3; ++sw)
      FL_CUDA(cudaFuncSetAttribute(sw == 2 ? pick_kernel_pair(ACT_NONE, epi->out_dtype)
                                           : pick_kernel(ACT_NONE, epi->out_dtype, sw == 1),
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, p.max_smem));
  }
  // the error word must start at zero; the intermediate is fully overwritten
  FL_CUDA(cudaMemsetAsync(p.d_err, 0, sizeof(int), reinterpret_cast<cudaStream_t>(stream_)));
  return fl_execute(&p, A, W, bias, aux, residual, out, stream_);
}
