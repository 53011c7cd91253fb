// fl_gemm.cuh — the fused linear layer as one persistent, warp-specialised
// tcgen05 kernel for sm_100a:
//
//     y = ((act(A·Wᵀ + bias)) + residual) · scale       [+ ReLU aux bitmask]
//
// The epilogue runs on the fp32 accumulator tile while it sits in tensor
// memory, so the GEMM result never makes an HBM round trip — the single
// launch / single write that the cuBLASLt epilog page ("通过 cuBLASLt 的
// epilog 机制实现单内核偏置融合") describes for RELU_BIAS / GELU_BIAS /
// RELU_AUX_BIAS, and the GEMM-epilogue fusion of the mHC page
// (mhpn.cn/news/2504128, §3.3).
//
// Roles (192 threads, one CTA per SM):
//   warp 0      TMA producer: A and B tiles into a multi-stage 128B-swizzled ring
//   warp 1      TMEM allocator + single-thread UMMA issuer (double-buffered accumulators)
//   warps 2..5  epilogue: tcgen05.ld → bias/act/aux/residual/scale in registers →
//               swizzled smem → TMA store (normal layout) or coalesced stores (swap-AB)
//
// Layouts:
//   * normal:  UMMA A = activation rows (128 per tile), UMMA B = weight rows;
//              TMEM lane = output row m, TMEM column = output column n.
//   * swap-AB (small M): UMMA A = weight rows (128 output features), UMMA B =
//              activation rows; TMEM lane = output column n, column = output row m.
//              Optional split-K across a thread-block cluster, reduced through
//              distributed shared memory BEFORE the (nonlinear) epilogue.
//
// Every wait is bounded (globaltimer); on expiry the kernel records an error
// code in a device word and unwinds: no trap, no unbounded spin.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fl_ptx.cuh"

// Phase-trace points (a device timestamp per CTA and slot).  Empty unless a trace
// build defines FL_STAMP before including this file.
#ifndef FL_STAMP
#define FL_STAMP(slot) \
  do {                 \
  } while (0)
#endif

namespace fl {

enum Act : int { ACT_NONE = 0, ACT_RELU = 1, ACT_GELU = 2, ACT_GELU_TANH = 3, ACT_GEGLU = 4, ACT_GELU_SIGMOID = 5 };
enum DType : int { DT_F16 = 0, DT_BF16 = 1, DT_F32 = 2 };

constexpr int kEpiWarp0 = 2;                 // warps 0,1: TMA producer, UMMA issuer
constexpr uint32_t kStagingBuf = 32 * 128;    // one epilogue warp's 32 rows x 128 bytes
constexpr int kUmmaSteps = 4;                 // UMMA instructions per 128-byte K atom
constexpr int kMaxSteps = 8;                  // at most two atoms per stage
constexpr int kErrTimeout = 1;

// 8 epilogue warps, two per TMEM lane quarter (the normal layout gives each a
// column half of the tile; the swap-AB layout a share of the rows).
template <bool SWAP>
struct Cfg {
  static constexpr int kEpiWarps = 8;
  static constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;
  static constexpr uint32_t kStagingBytes = SWAP ? 0u : kEpiWarps * kStagingBuf;
};

struct KParams {
  // output space: y is M x N
  int M, N, K;
  // MMA space
  int tiles_a, tiles_b;  // tiles along UMMA M (128 rows of operand A) / along UMMA N
  int num_kb;            // BK blocks along K
  int split_k;           // CTAs of a cluster sharing one tile along K (swap-AB only)
  int num_stages;
  int mma_n;             // UMMA N = TMEM columns per accumulator buffer
  int out_tile_n;        // output columns per tile in the normal layout (mma_n/2 for GeGLU)
  int bk;                // K elements per stage (128 bytes of operand)
  int b_boxes;           // TMA boxes of operand B per stage
  int b_box_rows;        // rows (K-major) or N-columns (MN-major) per B box
  int b_mn_major;        // 1: B stored [K, N]
  int geglu;             // 1: B = [gate rows ; up rows] from two tensor maps
  uint32_t a_stage_bytes, b_box_bytes, stage_bytes;  // stage_bytes: bytes one stage's TMA loads deliver
  uint32_t stage_stride;  // distance between stages (3xTF32 stages also hold the lo halves)
  int k_atoms;            // 128-byte swizzle atoms of K per stage (1, or 2 for 128-deep bf16 stages)
  uint32_t a_atom_bytes, b_atom_bytes;  // bytes of one atom of A / of (this CTA's) B
  int usteps;             // UMMA instructions per stage (4 per atom)
  uint32_t idesc;
  uint32_t a_kstep, b_kstep;  // descriptor start-address advance per UMMA K step (bytes)
  uint32_t b_lbo;             // leading byte offset of an MN-major B operand
  uint32_t tmem_cols;
  uint32_t staging_off, bias_off, bar_off, red_off, red_pitch;
  uint32_t res_off;        // swap-AB: per-warp residual staging (two 32-row blocks per warp)
  uint32_t res_blk_bytes;  // one 32-row x 32-column block of the residual
  int res_async;           // 1: the residual is staged by 16-byte cp.async (aligned rows)
  // epilogue operands
  const void* bias;
  int bias_dtype, bias_axis;
  const void* residual;
  long long ldr;
  int res_dtype;
  void* out;
  long long ldo;
  uint32_t* aux;
  long long ld_aux;
  float scale;
  int n_tma;  // columns [0, n_tma) go out by TMA store; n_tma·size is a multiple of 16 bytes
  int* err;
  unsigned long long wait_limit_ns;
  // stream-K: the last sk_tiles tiles of the tile order are split along K into
  // sk_clusters contiguous ranges of (tile, K-block) units (0: data-parallel only)
  int sk_tiles, sk_clusters;
  // the data-parallel tiles (all but the stream-K ones) over the launch's clusters:
  // quotient and remainder, so that a cluster's count needs no division on the device
  int dp_q, dp_r;
  float inv_group;  // 1 / (8 * tiles_b): the tile raster's group size, inverted on the host
  float* sk_ws;   // fp32 partial accumulators: [cluster][CTA rank][epilogue warp][mma_n/2 x 32]
  int* sk_flags;  // [cluster][CTA rank][epilogue warp]: 1 once that warp's partial is stored
};

// ------------------------------------------------------------------ work schedule
// A cluster's work is a sequence of items, the same for its producer, MMA and
// epilogue warps: first its data-parallel tiles (tile cluster, cluster + clusters, ...
// below dp_tiles = all tiles - sk_tiles, each over the K blocks [kb_a, kb_b)), then
// (stream-K) its contiguous range [s_c, s_c+1) of the units u = (tile - dp_tiles)·num_kb
// + kb of the remaining tiles, s_c = ⌊c·U/sk_clusters⌋.  A range cuts at most two
// tiles: its first segment may start inside a tile (PARTIAL: the accumulator is stored
// for that tile's finisher), its last segment may hold a tile's first K blocks without
// its last (FINISH: the partials of the following clusters w0..w1, whose ranges start
// inside the tile, are added in cluster order before the epilogue).  A finisher
// processes its segment last and its writers process theirs first, so it rarely waits.
enum ItemKind : int { IT_FULL = 0, IT_PARTIAL = 1, IT_FINISH = 2 };
struct Item {
  int tile, kb0, kb1, kind, w0, w1;
};
__host__ __device__ __forceinline__ int sk_start(const KParams& p, int c) {
  return (int)((long long)p.sk_tiles * p.num_kb * c / p.sk_clusters);
}
// dp_q, dp_r of a launch of `ncl` clusters and the raster's inverse group size (set on
// the host beside the grid).
__host__ __device__ inline void set_dp_split(KParams& p, int ncl) {
  const int dp_tiles = p.tiles_a * p.tiles_b - p.sk_tiles;
  p.dp_q = dp_tiles / ncl;
  p.dp_r = dp_tiles % ncl;
  p.inv_group = 1.0f / (float)(8 * (p.tiles_b > 0 ? p.tiles_b : 1));
}
// Item i of cluster `cl` (0 <= cl < ncl) of `ncl` (false past the last); data-parallel
// tiles cover the K blocks [kb_a, kb_b).  Stateless, so that a role keeps only its item
// counter live.  Cluster cl holds the data-parallel tiles cl, cl + ncl, ...: dp_q of
// them, one more when cl < dp_r.
__host__ __device__ __forceinline__ bool get_item(const KParams& p, int cl, int ncl, int kb_a, int kb_b, int i,
                                                  Item& it) {
  const int dp_tiles = p.tiles_a * p.tiles_b - p.sk_tiles;
  const int n_dp = p.dp_q + (cl < p.dp_r ? 1 : 0);
  it.w0 = 0;
  it.w1 = -1;
  if (i < n_dp) {
    it.tile = cl + i * ncl;
    it.kb0 = kb_a;
    it.kb1 = kb_b;
    it.kind = IT_FULL;
    return true;
  }
  if (cl >= p.sk_clusters) return false;
  const int nkb = p.num_kb;
  const int s = sk_start(p, cl), e = sk_start(p, cl + 1);
  const int j = i - n_dp;
  // segment j of the range: the first starts at s, the others at tile boundaries
  const int u = (j == 0) ? s : (s / nkb + j) * nkb;
  if (u >= e) return false;
  const int tl = u / nkb, ts = tl * nkb, te = ts + nkb;
  const int se = e < te ? e : te;
  it.tile = dp_tiles + tl;
  it.kb0 = u - ts;
  it.kb1 = se - ts;
  if (u == ts && se == te) {
    it.kind = IT_FULL;
  } else if (u > ts) {
    it.kind = IT_PARTIAL;
  } else {
    it.kind = IT_FINISH;
    it.w0 = cl + 1;
    it.w1 = cl;
    while (it.w1 + 1 < p.sk_clusters && sk_start(p, it.w1 + 1) < te) ++it.w1;
  }
  return true;
}

// ------------------------------------------------------------------ helpers
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, const KParams& p,
                                             bool cluster_scope = false) {
  if (cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t spins = 0;
  while (true) {
    if (cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
    if ((++spins & 63u) == 0 && globaltimer_ns() - t0 > p.wait_limit_ns) {
      atomicCAS(p.err, 0, kErrTimeout);
      return false;
    }
  }
}

// Position in the shared-memory ring: stage index and the parity of its current fill.
// Kept incrementally: the UMMA issuer's per-stage work between two batches of UMMAs
// leaves the tensor pipe idle (it queues little), and a division by the runtime stage
// count there costs more than a stage's barrier wait.
struct StageRing {
  uint32_t s = 0, ph = 0;
  __device__ __forceinline__ void next(uint32_t ns) {
    if (++s == ns) {
      s = 0;
      ph ^= 1u;
    }
  }
};

// Warp-uniform bounded wait: lane 0 spins, the verdict is broadcast.
__device__ __forceinline__ bool warp_wait_bounded(uint32_t bar, uint32_t parity, const KParams& p,
                                                  int lane, bool cluster_scope = false) {
  uint32_t ok = 0;
  if (lane == 0) ok = wait_bounded(bar, parity, p, cluster_scope) ? 1u : 0u;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) {
    // The phase has completed and cannot complete again before this warp
    // arrives elsewhere, so each lane's own test succeeds at once and gives
    // every lane the barrier's acquire ordering.
    if (cluster_scope) (void)mbar_try_wait_cluster(bar, parity);
    else (void)mbar_try_wait(bar, parity);
  }
  return ok != 0;
}

// Warp-uniform bounded wait until a GPU-scope flag in global memory is nonzero (set with
// release semantics by another CTA); every lane then acquires it itself.
__device__ __forceinline__ bool warp_wait_flag(const int* f, const KParams& p, int lane) {
  uint32_t ok = 1;
  if (lane == 0 && ld_acquire_gpu(f) == 0) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu(f) == 0) {
      if (globaltimer_ns() - t0 > p.wait_limit_ns) {
        atomicCAS(p.err, 0, kErrTimeout);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) (void)ld_acquire_gpu(f);
  return ok != 0;
}

// Stream-K workspace of one epilogue warp: its accumulator columns in blocks of 32
// columns x 32 rows; inside a block, float4 j4 of lane l (columns 4·j4 .. 4·j4+3 of row l)
// is at (j4·32 + l)·4, so a warp-wide float4 access covers 512 contiguous bytes.
__device__ __forceinline__ float* sk_area(const KParams& p, int cluster, int cta_rank, int kcl, int ew) {
  return p.sk_ws + ((size_t)(cluster * kcl + cta_rank) * 8u + (size_t)ew) * (size_t)(p.mma_n / 2) * 32u;
}
// x[0..31] += block `blk` of a stored partial (this lane's row)
__device__ __forceinline__ void sk_add_block(float* x, const float* area, int blk, int lane) {
  const float4* src = reinterpret_cast<const float4*>(area + (size_t)blk * 1024u) + lane;
#pragma unroll
  for (int j4 = 0; j4 < 8; ++j4) {
    const float4 q = __ldcg(src + j4 * 32);
    x[4 * j4] += q.x;
    x[4 * j4 + 1] += q.y;
    x[4 * j4 + 2] += q.z;
    x[4 * j4 + 3] += q.w;
  }
}

// Stream-K, out of line (taken at most twice per CTA, so the register-bound epilogue loop
// keeps its allocation): the warp's accumulator blocks b = 0 .. mma_n/64 - 1 sit at TMEM
// column c_begin + 32b, or, past gblk blocks (GeGLU's up half), out_tile_n + c_begin +
// 32(b - gblk).
__device__ __noinline__ void sk_store_partial(const KParams& p, uint32_t tacc, int c_begin, int gblk, float* area,
                                              int lane) {
#pragma unroll 1
  for (int b = 0; b < p.mma_n / 64; ++b) {
    const int col = b < gblk ? c_begin + 32 * b : p.out_tile_n + c_begin + 32 * (b - gblk);
    uint32_t r[32];
    tmem_ld32(tacc + (uint32_t)col, r);
    tmem_wait_ld();
    float4* dst = reinterpret_cast<float4*>(area + (size_t)b * 1024u) + lane;
#pragma unroll
    for (int j4 = 0; j4 < 8; ++j4)
      __stcg(dst + j4 * 32, make_float4(__uint_as_float(r[4 * j4]), __uint_as_float(r[4 * j4 + 1]),
                                        __uint_as_float(r[4 * j4 + 2]), __uint_as_float(r[4 * j4 + 3])));
  }
}
// acc += the partials of clusters w0..w1 (in that order), block by block in TMEM
__device__ __noinline__ void sk_add_partials(const KParams& p, uint32_t tacc, int c_begin, int gblk, int cta_rank,
                                             int kcl, int ew, int w0, int w1, int lane) {
#pragma unroll 1
  for (int b = 0; b < p.mma_n / 64; ++b) {
    const int col = b < gblk ? c_begin + 32 * b : p.out_tile_n + c_begin + 32 * (b - gblk);
    uint32_t r[32];
    tmem_ld32(tacc + (uint32_t)col, r);
    tmem_wait_ld();
    float x[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(r[j]);
#pragma unroll 1
    for (int w = w0; w <= w1; ++w) sk_add_block(x, sk_area(p, w, cta_rank, kcl, ew), b, lane);
#pragma unroll
    for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(x[j]);
    tmem_st32(tacc + (uint32_t)col, r);
  }
  tmem_wait_st();
}

__device__ __forceinline__ float load_elem(const void* p, long long i, int dt) {
  if (dt == DT_BF16) return __bfloat162float(__ldg(reinterpret_cast<const __nv_bfloat16*>(p) + i));
  if (dt == DT_F16) return __half2float(__ldg(reinterpret_cast<const __half*>(p) + i));
  return __ldg(reinterpret_cast<const float*>(p) + i);
}

template <int OUT>
__device__ __forceinline__ void store_elem(void* p, long long i, float v) {
  if constexpr (OUT == DT_BF16) {
    reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  } else if constexpr (OUT == DT_F16) {
    reinterpret_cast<__half*>(p)[i] = __float2half_rn(v);
  } else {
    reinterpret_cast<float*>(p)[i] = v;
  }
}

// erf by Abramowitz & Stegun, Handbook of Mathematical Functions, formula 7.1.26:
// with t = 1/(1 + p|x|), erf(|x|) = 1 - t(a1 + t(a2 + t(a3 + t(a4 + t·a5))))·e^(-x²),
// absolute error at most 1.5e-7; erf is odd.  e^(-x²) and 1/(1 + p|x|) come from the
// special-function unit (relative errors near 2^-22), which keeps the total error
// near 2e-7, far inside the fp32 tolerance of the layer.
// (erf_as_e also returns the e^(-x²) it used)
__device__ __forceinline__ float erf_as_e(float x, float& e) {
  const float ax = fabsf(x);
  const float t = rcp_approx(fmaf(0.3275911f, ax, 1.0f));
  float q = fmaf(1.061405429f, t, -1.453152027f);
  q = fmaf(q, t, 1.421413741f);
  q = fmaf(q, t, -0.284496736f);
  q = fmaf(q, t, 0.254829592f);
  q *= t;
  e = ex2_approx(-(ax * ax) * 1.4426950408889634f);  // e^(-x²)
  return copysignf(fmaf(-q, e, 1.0f), x);
}
__device__ __forceinline__ float erf_as(float x) {
  float e;
  return erf_as_e(x, e);
}
// tanh(u) = 1 - 2/(e^(2u) + 1): saturates to ±1 exactly (e^(2u) = inf or 0), absolute
// error near 2^-22 elsewhere.
__device__ __forceinline__ float tanh_ex2(float u) {
  const float e = ex2_approx(u * 2.8853900817779268f);  // e^(2u)
  return fmaf(-2.0f, rcp_approx(e + 1.0f), 1.0f);
}

// GELU(x) = x·Φ(x) = x/2·(1 + erf(x/√2))
__device__ __forceinline__ float gelu_erf_f(float x) {
  return 0.5f * x * (1.0f + erf_as(x * 0.70710678118654752f));
}
// GELU-tanh(x) = x/2·(1 + tanh(√(2/π)·(x + 0.044715x³))).  LOWP (16-bit outputs,
// relative precision 2^-8): tanh on the special-function unit (relative error
// about 2^-11); otherwise the exp-based form above.
template <bool LOWP>
__device__ __forceinline__ float gelu_tanh_f(float x) {
  const float u = 0.79788456080286536f * fmaf(0.044715f * x, x * x, x);
  return 0.5f * x * (1.0f + (LOWP ? tanh_approx(u) : tanh_ex2(u)));
}

// GELU's sigmoid form x·σ(1.702x) = x / (1 + 2^(-1.702·log2(e)·x)), reciprocal and
// power of two on the special-function unit (relative error near 2^-22)
__device__ __forceinline__ float gelu_sigmoid_f(float x) {
  return x * rcp_approx(1.0f + ex2_approx(-1.702f * 1.4426950408889634f * x));
}

template <int ACT, bool LOWP = false>
__device__ __forceinline__ float activate(float v, float u) {
  if constexpr (ACT == ACT_RELU) return fmaxf(v, 0.0f);
  if constexpr (ACT == ACT_GELU) return gelu_erf_f(v);
  if constexpr (ACT == ACT_GELU_TANH) return gelu_tanh_f<LOWP>(v);
  if constexpr (ACT == ACT_GEGLU) return gelu_tanh_f<LOWP>(v) * u;
  if constexpr (ACT == ACT_GELU_SIGMOID) return gelu_sigmoid_f(v);
  return v;
}

// Pack 32 fp32 values into 32 little-endian 32-bit words of OUT type
// (16-bit: two values per word → 64 values give 32 words; fp32: one per word).
template <int OUT>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  if constexpr (OUT == DT_BF16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

__host__ __device__ __forceinline__ void tile_coords(int t, const KParams& p, int& ta, int& tb) {
  // Grouped raster: 8 A-side tiles per group, B-side swept inside the group,
  // so concurrently resident CTAs share operand panels in L2.  No integer division on
  // the way (it runs at every tile boundary): the group index is t times the host's
  // inverse group size, truncated and corrected by one step either way (exact for
  // t < 2^24), and a full group of 8 splits r by shifts.
  constexpr int G = 8;
  const int group_size = G * p.tiles_b;
  int g = (int)((float)t * p.inv_group);
  if (g * group_size > t) --g;
  if ((g + 1) * group_size <= t) ++g;
  const int first = g * G;
  const int r = t - g * group_size;
  const int ga = p.tiles_a - first;
  if (ga >= G) {
    ta = first + (r & (G - 1));
    tb = r >> 3;
  } else {
    ta = first + r % ga;
    tb = r / ga;
  }
}

// Pinned read-only global loads: volatile with a memory clobber, so a batch of
// them stays ahead of the stores that follow and all are in flight together.
__device__ __forceinline__ float ldg_pinned(const void* base, long long i, int dt) {
  if (dt == DT_F32) {
    float v;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(reinterpret_cast<const float*>(base) + i) : "memory");
    return v;
  }
  unsigned short h;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(h) : "l"(reinterpret_cast<const uint16_t*>(base) + i) : "memory");
  if (dt == DT_BF16) return __uint_as_float(static_cast<uint32_t>(h) << 16);
  return __half2float(__ushort_as_half(h));
}

// ------------------------------------------------------------------ failure-path self-test
// One thread waits, with the same bounded wait as the kernels, on an mbarrier that
// nothing arrives on: the wait gives up after `limit_ns`, records kErrTimeout in
// *err and the kernel returns, leaving the context usable.
__global__ void fl_wait_selftest_kernel(int* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_mbarrier_init();
  KParams p{};
  p.err = err;
  p.wait_limit_ns = limit_ns;
  (void)wait_bounded(b, 0, p);
}

// ------------------------------------------------------------------ 3xTF32 split
// x = hi + lo.  The tensor core reads a 32-bit operand word as TF32 by keeping its
// top 19 bits (sign, exponent, 10 mantissa bits): the raw stage word therefore
// serves as hi = trunc(x), and only lo = x - hi (exact in fp32, at most 13
// significant bits) is written, rounded to TF32 so that the tensor core reads it
// exactly.  x·y ≈ hi_x·hi_y + hi_x·lo_y + lo_x·hi_y.  (A reader that rounded
// instead of truncating would leave errors near 2^-11 per product, which the
// parity tests on inputs with all low bits set reject.)
__device__ __forceinline__ uint32_t tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ uint32_t tf32_lo(float x) {
  return tf32_rna(x - __uint_as_float(__float_as_uint(x) & 0xFFFFE000u));
}

// ------------------------------------------------------------------ epilogue helpers
// Store CH values of one row (first column nc0, element offset i0 of the row start)
// in OUT type: 16-byte vectors when the whole chunk lies inside the N columns (the
// caller's pitch and base are 16-byte aligned), else element by element up to N.
template <int OUT, int CH>
__device__ __forceinline__ void store_row_chunk(void* base, long long i0, int nc0, int N, const float (&v)[CH]) {
  constexpr int ES = (OUT == DT_F32) ? 4 : 2;
  if (nc0 + CH <= N) {
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<char*>(base) + i0 * ES);
#pragma unroll
    for (int c = 0; c < CH * ES / 16; ++c) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if constexpr (OUT == DT_F32) w[k] = __float_as_uint(v[4 * c + k]);
        else w[k] = pack2<OUT>(v[8 * c + 2 * k], v[8 * c + 2 * k + 1]);
      }
      dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < CH; ++j)
      if (nc0 + j < N) store_elem<OUT>(base, i0 + j, v[j]);
  }
}

// Load CH consecutive elements of one row (16-byte vectors when the whole chunk
// is in range, else guarded scalars) and widen them to fp32.
template <int CH>
__device__ __forceinline__ void load_row_chunk(float (&dst)[CH], const void* base, long long row_off, int n0,
                                               int N, int dt, bool full) {
  if (full) {
    if (dt == DT_F32) {
      const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + row_off + n0);
#pragma unroll
      for (int i = 0; i < CH / 4; ++i) {
        const float4 f = __ldg(src + i);
        dst[4 * i] = f.x;
        dst[4 * i + 1] = f.y;
        dst[4 * i + 2] = f.z;
        dst[4 * i + 3] = f.w;
      }
    } else {
      const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(base) + row_off + n0);
#pragma unroll
      for (int i = 0; i < CH / 8; ++i) {
        const uint4 u = __ldg(src + i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (dt == DT_BF16) {
            dst[8 * i + 2 * e] = __uint_as_float(w[e] << 16);
            dst[8 * i + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
          } else {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
            dst[8 * i + 2 * e] = f.x;
            dst[8 * i + 2 * e + 1] = f.y;
          }
        }
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      dst[j] = 0.0f;
      if (n0 + j < N) dst[j] = ldg_pinned(base, row_off + n0 + j, dt);
    }
  }
}

// CH consecutive 16-bit elements of a row, from element offset i0, kept as raw 16-byte
// vectors (two elements a 32-bit word, low half first).  Pinned volatile loads, so that
// they are issued here, ahead of their use; a chunk that ends past n_end (ragged row
// end) is read element by element, with zeros past n_end.  Requires 16-byte aligned
// rows when the chunk is whole.
template <int CH>
__device__ __forceinline__ void prefetch_row16(uint4 (&q)[CH / 8], const void* base, long long i0, int n0, int n_end) {
  const uint16_t* b = reinterpret_cast<const uint16_t*>(base) + i0;
  if (n0 + CH <= n_end) {
#pragma unroll
    for (int i = 0; i < CH / 8; ++i)
      asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(q[i].x), "=r"(q[i].y), "=r"(q[i].z), "=r"(q[i].w)
                   : "l"(b + 8 * i)
                   : "memory");
  } else {
#pragma unroll
    for (int i = 0; i < CH / 8; ++i) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t lo = 0, hi = 0;
        const int j = 8 * i + 2 * k;
        if (n0 + j < n_end) {
          unsigned short h;
          asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(h) : "l"(b + j) : "memory");
          lo = h;
        }
        if (n0 + j + 1 < n_end) {
          unsigned short h;
          asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(h) : "l"(b + j + 1) : "memory");
          hi = h;
        }
        w[k] = lo | (hi << 16);
      }
      q[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}
// element j of a chunk prefetched by prefetch_row16, widened to fp32
__device__ __forceinline__ float row16_elem(const uint4* q, int j, int dt) {
  const uint4 v = q[j >> 3];
  const int k = (j >> 1) & 3;
  const uint32_t w = k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
  const uint32_t h = (j & 1) ? (w >> 16) : (w & 0xFFFFu);
  return dt == DT_BF16 ? __uint_as_float(h << 16) : __half2float(__ushort_as_half((unsigned short)h));
}

// Eight read-only loads base[i0], base[i0+stride], ... issued by one asm
// statement, so all eight are in flight before any result is used.  Every
// address must be valid (callers clamp the row index).
__device__ __forceinline__ void ldg8(float (&dst)[8], const void* base, long long i0, long long stride, int dt) {
  if (dt == DT_F32) {
    const float* b = reinterpret_cast<const float*>(base) + i0;
    asm volatile(
        "ld.global.nc.f32 %0, [%8];\n\tld.global.nc.f32 %1, [%9];\n\tld.global.nc.f32 %2, [%10];\n\t"
        "ld.global.nc.f32 %3, [%11];\n\tld.global.nc.f32 %4, [%12];\n\tld.global.nc.f32 %5, [%13];\n\t"
        "ld.global.nc.f32 %6, [%14];\n\tld.global.nc.f32 %7, [%15];"
        : "=f"(dst[0]), "=f"(dst[1]), "=f"(dst[2]), "=f"(dst[3]), "=f"(dst[4]), "=f"(dst[5]), "=f"(dst[6]),
          "=f"(dst[7])
        : "l"(b), "l"(b + stride), "l"(b + 2 * stride), "l"(b + 3 * stride), "l"(b + 4 * stride),
          "l"(b + 5 * stride), "l"(b + 6 * stride), "l"(b + 7 * stride)
        : "memory");
    return;
  }
  const uint16_t* b = reinterpret_cast<const uint16_t*>(base) + i0;
  unsigned short h[8];
  asm volatile(
      "ld.global.nc.u16 %0, [%8];\n\tld.global.nc.u16 %1, [%9];\n\tld.global.nc.u16 %2, [%10];\n\t"
      "ld.global.nc.u16 %3, [%11];\n\tld.global.nc.u16 %4, [%12];\n\tld.global.nc.u16 %5, [%13];\n\t"
      "ld.global.nc.u16 %6, [%14];\n\tld.global.nc.u16 %7, [%15];"
      : "=h"(h[0]), "=h"(h[1]), "=h"(h[2]), "=h"(h[3]), "=h"(h[4]), "=h"(h[5]), "=h"(h[6]), "=h"(h[7])
      : "l"(b), "l"(b + stride), "l"(b + 2 * stride), "l"(b + 3 * stride), "l"(b + 4 * stride),
        "l"(b + 5 * stride), "l"(b + 6 * stride), "l"(b + 7 * stride)
      : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i)
    dst[i] = (dt == DT_BF16) ? __uint_as_float(static_cast<uint32_t>(h[i]) << 16) : __half2float(__ushort_as_half(h[i]));
}

// Swap-AB epilogue, residual staging: rows [m0, m0+cnt) x columns [n0, n0+32)
// of the residual go to shared memory (row-major, 32 elements a row) by 16-byte
// cp.async, one commit group per call.  Bytes past column N are zero-filled;
// every row copied is below M.  Requires 16-byte aligned rows (res_async).
__device__ __forceinline__ void stage_residual(const KParams& p, uint32_t dst, int m0, int cnt, int n0, int lane) {
  const int es = (p.res_dtype == DT_F32) ? 4 : 2;
  const int cpr = 2 * es;  // 16-byte chunks in a 32-element row
  const char* base = reinterpret_cast<const char*>(p.residual);
#pragma unroll 1
  for (int c = lane; c < cnt * cpr; c += 32) {
    const int r = c / cpr, k = c - r * cpr;
    const int col = n0 + k * (16 / es);
    const int bytes = min(max(p.N - col, 0) * es, 16);
    const char* src = bytes > 0 ? base + ((long long)(m0 + r) * p.ldr + col) * es : base;
    cp_async_16(dst + (uint32_t)(r * 32 * es + k * 16), src, (uint32_t)bytes);
  }
  cp_async_commit();
}

// ------------------------------------------------------------------ kernel
template <int ACT, int OUT, bool SWAP, bool TF32 = false, bool PAIR = false>
__global__ void __launch_bounds__(Cfg<SWAP>::kThreads, 1)
    fl_gemm_epi_tcgen05(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmOut,
                        const __grid_constant__ KParams p) {
  constexpr int kEpiWarps = Cfg<SWAP>::kEpiWarps;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t smem_base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int NS = p.num_stages;

  const uint32_t bars = smem_base + p.bar_off;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (NS + s); };
  auto tfull_bar = [&](int b) { return bars + 8u * (2 * NS + b); };
  auto tempty_bar = [&](int b) { return bars + 8u * (2 * NS + 2 + b); };
  const uint32_t drain_bar = bars + 8u * (2 * NS + 4);
  const uint32_t red_ready_bar = bars + 8u * (2 * NS + 5);
  const uint32_t red_done_bar = bars + 8u * (2 * NS + 6);
  const uint32_t tmem_slot = bars + 8u * (2 * NS + 7);
  auto conv_bar = [&](int s) { return bars + 8u * (2 * NS + 8 + s); };  // 3xTF32: stage split done
  // swap-AB split-K: the partial slices that the peers push (the slot of the first
  // 3xTF32 barrier, which that layout does not use)
  const uint32_t recv_bar = bars + 8u * (2 * NS + 8);

  // Clusters: split-K groups of S CTAs (swap layout), or CTA pairs that share one
  // 256-row UMMA (PAIR: rank 0 issues the UMMA for both, each CTA owns 128 rows).
  const int S = p.split_k;
  constexpr int kCl = PAIR ? 2 : 1;
  const uint32_t rank = (S > 1 || PAIR) ? cluster_ctarank() : 0u;
  const int csize = PAIR ? kCl : S;
  const int cluster_id = blockIdx.x / csize;
  const int num_clusters = gridDim.x / csize;
  const uint32_t krank = PAIR ? 0u : rank;  // split-K slice of this CTA
  const int kb_begin = (int)(((long long)p.num_kb * krank) / S);
  const int kb_end = (int)(((long long)p.num_kb * (krank + 1)) / S);
  const int tile_rows = PAIR ? 256 : 128;   // output rows per tile (both CTAs of a pair)
  const int cta_row_off = PAIR ? (int)rank * 128 : 0;

  if (threadIdx.x == 0) {
    FL_STAMP(0);
    for (int s = 0; s < NS; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), kEpiWarps * kCl);  // PAIR: the peer's epilogue warps arrive too
    }
    mbar_init(drain_bar, 1);
    // split-K hand-off: one arrive per epilogue warp (after __syncwarp, so the
    // release covers the whole warp's shared-memory writes)
    mbar_init(red_ready_bar, kEpiWarps * S);
    mbar_init(red_done_bar, S - 1 > 0 ? S - 1 : 1);  // one arrival per peer that received our slices
    if (SWAP && S > 1) mbar_init(recv_bar, 1);
    if (TF32)  // PAIR: both CTAs' converters arrive on the leader's barrier
      for (int s = 0; s < NS; ++s) mbar_init(conv_bar(s), kEpiWarps * kCl);
    fence_mbarrier_init();
    if (p.num_kb > 0) {  // with K = 0 the operand maps are left unencoded and never used
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmB);
      if (p.geglu) prefetch_tensormap(&tmB2);
    }
    if (!SWAP) prefetch_tensormap(&tmOut);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, p.tmem_cols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, p.tmem_cols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (S > 1 || PAIR) cluster_sync_all();  // peers' barriers are initialised before any remote arrive
  if (threadIdx.x == 0) FL_STAMP(1);
  // Programmatic dependent launch: the prologue above may overlap the previous
  // kernel of the stream; no global memory is touched before this wait.
  grid_dependency_wait();
  if (threadIdx.x == 0) {
    FL_STAMP(2);
    grid_launch_dependents();
  }
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(
      __cvta_shared_to_generic(tmem_slot));

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      StageRing rs;
      bool ok = true;
      Item itm;
      for (int ii = 0; ok && get_item(p, cluster_id, num_clusters, kb_begin, kb_end, ii, itm); ++ii) {
        int ta, tb;
        tile_coords(itm.tile, p, ta, tb);
        const int a_row = ta * tile_rows + cta_row_off;
        // PAIR: each CTA loads its half of the B tile
        const int b_row = tb * p.mma_n + (PAIR ? (int)rank * (p.mma_n / 2) : 0);
        const int g_row = tb * p.b_box_rows;
        for (int kb = itm.kb0; kb < itm.kb1; ++kb, ++it, rs.next((uint32_t)NS)) {
          const int s = (int)rs.s;
          const uint32_t ph = rs.ph;
          if (!wait_bounded(empty_bar(s), ph ^ 1u, p)) { ok = false; break; }
          if (it == 0) FL_STAMP(3);
          const uint32_t sa = smem_base + (uint32_t)s * p.stage_stride;
          const uint32_t sb = sa + p.a_stage_bytes;
          const int k0 = kb * p.bk;
          const int ae = p.bk / p.k_atoms;  // K elements of one 128-byte atom
          if constexpr (PAIR && !TF32) {
            // both CTAs' bytes complete on the leader's full barrier
            const uint32_t fb = mapa_shared(full_bar(s), 0);
            if (rank == 0) mbar_arrive_expect_tx(full_bar(s), 2u * p.stage_bytes);
            for (int a = 0; a < p.k_atoms; ++a)
              tma_load_2d_pair(sa + a * p.a_atom_bytes, &tmA, fb, k0 + a * ae, a_row);
            if (p.b_mn_major) {
              for (int i = 0; i < p.b_boxes; ++i)
                tma_load_2d_pair(sb + i * p.b_box_bytes, &tmB, fb, b_row + i * 64, k0);
            } else {
              // GeGLU: the pair's 256-wide B tile is [128 gate rows (rank 0) ; 128 up rows (rank 1)]
              const CUtensorMap* mb = (p.geglu && rank != 0) ? &tmB2 : &tmB;
              const int br = p.geglu ? g_row : b_row;
              for (int a = 0; a < p.k_atoms; ++a) tma_load_2d_pair(sb + a * p.b_atom_bytes, mb, fb, k0 + a * ae, br);
            }
          } else {
            const uint32_t fb = full_bar(s);
            mbar_arrive_expect_tx(fb, p.stage_bytes);
            for (int a = 0; a < p.k_atoms; ++a) tma_load_2d(sa + a * p.a_atom_bytes, &tmA, fb, k0 + a * ae, a_row);
            if (p.b_mn_major) {
              // one box covers the stage's bk rows of the N-contiguous B
              for (int i = 0; i < p.b_boxes; ++i) tma_load_2d(sb + i * p.b_box_bytes, &tmB, fb, b_row + i * 64, k0);
            } else if (p.geglu) {
              for (int a = 0; a < p.k_atoms; ++a) {
                tma_load_2d(sb + a * p.b_atom_bytes, &tmB, fb, k0 + a * ae, g_row);
                tma_load_2d(sb + a * p.b_atom_bytes + p.b_box_bytes, &tmB2, fb, k0 + a * ae, g_row);
              }
            } else {
              for (int a = 0; a < p.k_atoms; ++a)
                for (int i = 0; i < p.b_boxes; ++i)
                  tma_load_2d(sb + a * p.b_atom_bytes + i * p.b_box_bytes, &tmB, fb, k0 + a * ae,
                              b_row + i * p.b_box_rows);
            }
          }
        }
      }
      // Never leave the CTA with copies in flight: wait (bounded) for the last
      // fill of every stage (fill i went to stage i % NS with phase (i / NS) & 1).
      // In the normal path these have all completed already.  A pair's peer
      // counts its bytes on the leader's barriers, which the leader waits for; the
      // final cluster barrier keeps the peer resident until then.
      for (uint32_t s = 0; (!PAIR || TF32 || rank == 0) && s < (uint32_t)NS && s < it; ++s) {
        const uint32_t last = it - 1u - ((it - 1u - s) % (uint32_t)NS);
        (void)wait_bounded(full_bar((int)s), (last / (uint32_t)NS) & 1u, p);
      }
    }
    __syncwarp();  // reconverge: the CTA barrier below is warp-aligned
  } else if (warp == 1) {
    // ================================================================ UMMA issuer
    if (lane == 0 && (!PAIR || rank == 0)) {  // in a pair, rank 0 issues for both CTAs
      // Descriptors of stage 0; a stage s and UMMA step k only move the start
      // address field (addresses stay below 2^18 bytes, so no carry leaves it).
      const uint64_t da0 = sdesc_sw128(smem_base, 16, 1024);
      const uint64_t db0 = sdesc_sw128(smem_base + p.a_stage_bytes, p.b_mn_major ? p.b_lbo : 16u, 1024);
      const uint64_t stage_step = p.stage_stride >> 4;
      // 3xTF32: lo halves of A and B follow the raw (hi) tiles inside each stage
      const uint32_t lo_off = p.stage_bytes;
      const uint64_t dal0 = sdesc_sw128(smem_base + lo_off, 16, 1024);
      const uint64_t dbl0 = sdesc_sw128(smem_base + lo_off + p.a_stage_bytes, 16, 1024);
      const uint64_t ak = p.a_kstep >> 4, bk = p.b_kstep >> 4;
      // start-address offsets (16-byte units) of UMMA step j inside a stage: atom j/4,
      // then 32 bytes per step inside the atom (an MN-major B advances 16 K rows per step)
      uint32_t aso[kMaxSteps], bso[kMaxSteps];
#pragma unroll
      for (int j = 0; j < kMaxSteps; ++j) {
        aso[j] = ((uint32_t)(j >> 2) * p.a_atom_bytes + (uint32_t)(j & 3) * p.a_kstep) >> 4;
        bso[j] = p.b_mn_major ? ((uint32_t)j * p.b_kstep) >> 4
                              : ((uint32_t)(j >> 2) * p.b_atom_bytes + (uint32_t)(j & 3) * p.b_kstep) >> 4;
      }
      const int usteps = p.usteps;
      const uint32_t idesc = p.idesc;
      uint32_t it = 0, local = 0;
      StageRing rs;
      bool ok = true, issued = false;
      Item itm;
      for (; ok && get_item(p, cluster_id, num_clusters, kb_begin, kb_end, (int)local, itm); ++local) {
        const bool acc_any = itm.kb1 > itm.kb0;
        const uint32_t buf = local & 1u;
        const uint32_t tph = (local >> 1) & 1u;
        if (!wait_bounded(tempty_bar(buf), tph ^ 1u, p, PAIR)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * (uint32_t)p.mma_n;
        for (int kb = itm.kb0; kb < itm.kb1; ++kb, ++it, rs.next((uint32_t)NS)) {
          const int s = (int)rs.s;
          const uint32_t ph = rs.ph;
          if (!wait_bounded(TF32 ? conv_bar(s) : full_bar(s), ph, p, TF32 && PAIR)) { ok = false; break; }
          tc_fence_after();
          if (it == 0) FL_STAMP(4);
          const uint64_t da = da0 + (uint64_t)s * stage_step;
          const uint64_t db = db0 + (uint64_t)s * stage_step;
          if constexpr (TF32) {
            const uint64_t dal = dal0 + (uint64_t)s * stage_step;
            const uint64_t dbl = dbl0 + (uint64_t)s * stage_step;
#pragma unroll
            for (int k = 0; k < kUmmaSteps; ++k) {
              if constexpr (PAIR) {
                umma_tf32_pair(d_tmem, dal + k * ak, db + k * bk, idesc, (kb > itm.kb0 || k > 0) ? 1u : 0u);
                umma_tf32_pair(d_tmem, da + k * ak, dbl + k * bk, idesc, 1u);
                umma_tf32_pair(d_tmem, da + k * ak, db + k * bk, idesc, 1u);
              } else {
                umma_tf32(d_tmem, dal + k * ak, db + k * bk, idesc, (kb > itm.kb0 || k > 0) ? 1u : 0u);
                umma_tf32(d_tmem, da + k * ak, dbl + k * bk, idesc, 1u);
                umma_tf32(d_tmem, da + k * ak, db + k * bk, idesc, 1u);
              }
            }
          } else if constexpr (PAIR) {
#pragma unroll
            for (int k = 0; k < kMaxSteps; ++k)
              if (k < usteps)
                umma_f16_pair(d_tmem, da + aso[k], db + bso[k], idesc, (kb > itm.kb0 || k > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int k = 0; k < kMaxSteps; ++k)
              if (k < usteps)
                umma_f16(d_tmem, da + aso[k], db + bso[k], idesc, (kb > itm.kb0 || k > 0) ? 1u : 0u);
          }
          if constexpr (PAIR) {  // free the stage in both CTAs once these MMAs have read it
            umma_commit_pair_both(empty_bar(s));
          } else {
            umma_commit(empty_bar(s));  // frees the stage once these MMAs have read it
          }
          issued = true;
        }
        if (!ok) break;
        if (local == 0) FL_STAMP(5);
        if constexpr (PAIR) {
          if (acc_any) {
            umma_commit_pair_both(tfull_bar(buf));
          } else {
            mbar_arrive(tfull_bar(buf));
            mbar_arrive_remote(mapa_shared(tfull_bar(buf), 1));
          }
        } else {
          if (acc_any) umma_commit(tfull_bar(buf));
          else mbar_arrive(tfull_bar(buf));
        }
      }
      if (issued) {  // no MMA may still be running when TMEM is released
        if constexpr (PAIR) umma_commit_pair(drain_bar);
        else umma_commit(drain_bar);
        (void)wait_bounded(drain_bar, 0, p);
      }
    }
    __syncwarp();  // reconverge: the CTA barrier below is warp-aligned
  } else {
    // ================================================================ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int ew = warp - kEpiWarp0;
    const float scale = p.scale;
    const bool has_bias = p.bias != nullptr;
    const bool has_res = p.residual != nullptr;
    const bool has_aux = p.aux != nullptr;
    const bool has_mask = has_aux && ACT != ACT_GELU;  // the ReLU mask (GELU_AUX stores v instead)
    uint32_t local = 0;
    bool ok = true;

    if constexpr (!SWAP) {
      // ---------------- normal layout: thread = output row, a warp owns half the tile's columns
      constexpr int CH = (OUT == DT_F32) ? 32 : 64;  // output columns per 128-byte staging row
      const int half = ew >> 2;
      const uint32_t stg = smem_base + p.staging_off + (uint32_t)ew * kStagingBuf;
      const int half_cols = p.out_tile_n >> 1;
      StageRing crs;  // 3xTF32: ring position, in step with the producer and the MMA warp
      Item itm;
      for (; get_item(p, cluster_id, num_clusters, kb_begin, kb_end, (int)local, itm); ++local) {
        int ta, tb;
        tile_coords(itm.tile, p, ta, tb);
        const bool acc_any = itm.kb1 > itm.kb0;
        if constexpr (TF32) {
          // write the TF32 lo half of every stage of this tile beside it (the raw words
          // serve as hi); the 256 epilogue threads share the stage's 16-byte words
          const int et = (warp - kEpiWarp0) * 32 + lane;
          const uint32_t words = p.stage_bytes >> 4;
          for (int kb = itm.kb0; ok && kb < itm.kb1; ++kb, crs.next((uint32_t)NS)) {
            const int s = (int)crs.s;
            const uint32_t ph = crs.ph;
            if (!warp_wait_bounded(full_bar(s), ph, p, lane)) { ok = false; break; }
            const uint32_t st0 = smem_base + (uint32_t)s * p.stage_stride;
            for (uint32_t w = (uint32_t)et; w < words; w += kEpiWarps * 32) {
              const uint32_t a = st0 + 16u * w;
              float4 x;
              asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                           : "=f"(x.x), "=f"(x.y), "=f"(x.z), "=f"(x.w)
                           : "r"(a)
                           : "memory");
              const uint32_t l0 = tf32_lo(x.x), l1 = tf32_lo(x.y), l2 = tf32_lo(x.z), l3 = tf32_lo(x.w);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a + p.stage_bytes), "r"(l0), "r"(l1),
                           "r"(l2), "r"(l3)
                           : "memory");
            }
            fence_proxy_async_smem();  // the tensor core reads these through the async proxy
            __syncwarp();
            if (lane == 0) {
              // a pair's UMMA is issued by the leader: both CTAs' halves must be split
              if (PAIR && rank != 0) mbar_arrive_remote(mapa_shared(conv_bar(s), 0));
              else mbar_arrive(conv_bar(s));
            }
          }
          if (!ok) break;
        }
        const uint32_t buf = local & 1u;
        const uint32_t tph = (local >> 1) & 1u;
        const int row0 = ta * tile_rows + cta_row_off + q * 32;
        const int m = row0 + lane;
        const bool m_ok = m < p.M;
        const int n_tile0 = tb * p.out_tile_n;
        const int c_begin = half * half_cols;
        const int c_end = c_begin + half_cols;
        // ---- operands that do not depend on the accumulator, read before its barrier so
        // that their latency overlaps the main loop: the bias (per row; or lane l holds the
        // bias of columns c_begin + 32h + l of the tile), and the first chunk of a 16-bit
        // residual, as raw vectors (later chunks are read one chunk ahead)
        float bias_m = 0.0f;
        if (has_bias && p.bias_axis == 1 && m_ok) bias_m = ldg_pinned(p.bias, m, p.bias_dtype);
        float bias4[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int n = n_tile0 + c_begin + 32 * h + lane;
          bias4[h] = 0.0f;
          if (has_bias && p.bias_axis == 0 && 32 * h < half_cols && n < p.N) bias4[h] = ldg_pinned(p.bias, n, p.bias_dtype);
        }
        // (a 64-column chunk's prefetch buffer would not fit the register budget: those read
        // their residual at the start of the chunk)
        const bool res16 = CH == 32 && has_res && p.res_dtype != DT_F32;
        uint4 rq[CH / 8];
        if (res16 && m_ok && itm.kind != IT_PARTIAL)
          prefetch_row16<CH>(rq, p.residual, (long long)m * p.ldr + n_tile0 + c_begin, n_tile0 + c_begin, p.N);
        if (!warp_wait_bounded(tfull_bar(buf), tph, p, lane, PAIR)) { ok = false; break; }
        tc_fence_after();
        if (ew == 0 && lane == 0) {
          if (local == 0) FL_STAMP(6);
          FL_STAMP(8);
        }
        const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + buf * (uint32_t)p.mma_n;
        const int gblk = half_cols / 32;  // 32-column blocks of this warp's (gate) columns
        if (itm.kind == IT_PARTIAL) {
          // stream-K: this cluster's range starts inside the tile.  Store this warp's fp32
          // accumulator columns for the tile's finisher, free the TMEM buffer, then release
          // the warp's flag (every lane's stores are fenced before it).
          sk_store_partial(p, tacc, c_begin, gblk, sk_area(p, cluster_id, (int)rank, kCl, ew), lane);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (PAIR && rank != 0) mbar_arrive_remote(mapa_shared(tempty_bar(buf), 0));
            else mbar_arrive(tempty_bar(buf));
          }
          __threadfence();
          __syncwarp();
          if (lane == 0) st_release_gpu(p.sk_flags + (cluster_id * kCl + (int)rank) * kEpiWarps + ew, 1);
          if (ew == 0 && lane == 0) FL_STAMP(18);
          continue;
        }
        if (itm.kind == IT_FINISH) {
          // stream-K: add the partials of the clusters whose ranges start inside this tile
          // (in cluster order) to this warp's accumulator columns in tensor memory; the
          // epilogue below then reads the whole tile's sums
          for (int w = itm.w0; ok && w <= itm.w1; ++w)
            if (!warp_wait_flag(p.sk_flags + (w * kCl + (int)rank) * kEpiWarps + ew, p, lane)) ok = false;
          if (!ok) break;
          if (ew == 0 && lane == 0) FL_STAMP(16);
          sk_add_partials(p, tacc, c_begin, gblk, (int)rank, kCl, ew, itm.w0, itm.w1, lane);
          if (ew == 0 && lane == 0) FL_STAMP(17);
          // every lane has read the partials: the flags are ready for the next launch
          __syncwarp();
          if (lane == 0)
            for (int w = itm.w0; w <= itm.w1; ++w) p.sk_flags[(w * kCl + (int)rank) * kEpiWarps + ew] = 0;
        }

        // The warp's columns as 32-column blocks in a rolled loop: a block's accumulator,
        // bias, activation, mask, residual and scale live in 32 registers, and its packed
        // values go straight into the 128B-swizzled staging row of its chunk (CH columns,
        // 128 bytes a row), which leaves by one TMA store once its last block is in.  The
        // next block's TMEM read is issued before this block's arithmetic, so its latency
        // overlaps it.
        constexpr int GPB = (OUT == DT_F32) ? 8 : 4;  // 16-byte granules per 32-column block
        constexpr int BPC = CH / 32;                  // blocks per chunk
        const int nblk = (c_end - c_begin) / 32;
        uint32_t ga[32], gu[32];  // the block's accumulator (GeGLU: gate and up columns)
        if (acc_any) {
          tmem_ld32(tacc + (uint32_t)c_begin, ga);
          if constexpr (ACT == ACT_GEGLU) tmem_ld32(tacc + (uint32_t)(p.out_tile_n + c_begin), gu);
          tmem_wait_ld();
        }
#pragma unroll 1
        for (int b = 0; b < nblk; ++b) {
          const int hh = b % BPC;
          const int cc = c_begin + 32 * (b - hh);  // first column of the block's chunk
          const int cb = c_begin + 32 * b;         // TMEM column (and tile column) of the block
          const int nc0 = n_tile0 + cc;
          const int n0 = n_tile0 + cb;              // the block's first output column
          // a chunk that reaches past this warp's columns (a 192-wide tile's last 32 columns of
          // a 16-bit output) is not stored by TMA: its 64-column box would cover the other
          // warp's columns.  Its block goes out by 16-byte stores from registers.
          const bool full_chunk = cc + CH <= c_end;
          const bool tma_chunk = nc0 < p.n_tma && full_chunk;
          if (hh == 0 && tma_chunk) {
            if (lane == 0) bulk_wait_group_read<0>();  // the previous store has read the staging row
            if (ew == 0 && lane == 0 && b == 0) FL_STAMP(25);
            __syncwarp();
          }
          const bool full32 = n0 + 32 <= p.N;
          const float blk_bias = b == 0 ? bias4[0] : b == 1 ? bias4[1] : b == 2 ? bias4[2] : bias4[3];
          // ---- accumulator of this block; the next block's read goes out now
          float v[32];
          if (acc_any) {
            if constexpr (ACT == ACT_GEGLU) {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = activate<ACT, OUT != DT_F32>(__uint_as_float(ga[j]), __uint_as_float(gu[j]));
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(ga[j]);
            }
            if (b + 1 < nblk) {
              tmem_ld32(tacc + (uint32_t)(cb + 32), ga);
              if constexpr (ACT == ACT_GEGLU) tmem_ld32(tacc + (uint32_t)(p.out_tile_n + cb + 32), gu);
            }
            if (ew == 0 && lane == 0 && b == 0) FL_STAMP(19);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = (ACT == ACT_GEGLU) ? activate<ACT, OUT != DT_F32>(0.0f, 0.0f) : 0.0f;
          }
          // ---- bias, activation, aux, residual, scale (all in fp32 registers)
          if (has_bias) {
            if (p.bias_axis == 0) {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] += __shfl_sync(0xffffffffu, blk_bias, j);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] += bias_m;
            }
          }
          if (ew == 0 && lane == 0 && hh == 0) {
            if (b == 0) FL_STAMP(23);
            if (b == BPC) FL_STAMP(27);
          }
          if constexpr (ACT == ACT_GELU) {
            // GELU_AUX_BIAS: the pre-activation v, in the output type, for the backward pass
            if (has_aux && m_ok) store_row_chunk<OUT, 32>(p.aux, (long long)m * p.ldo + n0, n0, p.N, v);
          }
          if (has_mask) {
            // bit j = (v_j > 0), in four independent partial words (the OR chains stay
            // short); the columns past N are cleared once for the whole word
            uint32_t w4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int j = 0; j < 32; ++j) w4[j & 3] |= (v[j] > 0.0f ? 1u : 0u) << j;
            uint32_t word = (w4[0] | w4[1]) | (w4[2] | w4[3]);
            if (!full32) {
              const int rem = p.N - n0;  // columns of the word inside the matrix, < 32
              word = rem > 0 ? word & ((1u << rem) - 1u) : 0u;
            }
            if (m_ok && (long long)n0 < p.N) p.aux[(long long)m * p.ld_aux + (n0 >> 5)] = word;
          }
          if constexpr (ACT != ACT_GEGLU) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = activate<ACT, OUT != DT_F32>(v[j], 0.0f);
          }
          if (has_res && m_ok) {
            if (res16) {
              // (res16: 32-column chunks, one block a chunk)
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] += row16_elem(rq, j, p.res_dtype);
              // the next chunk's residual travels while this chunk is stored
              if (b + 1 < nblk) prefetch_row16<CH>(rq, p.residual, (long long)m * p.ldr + n0 + 32, n0 + 32, p.N);
            } else {
              // (an fp32 residual, or 64-column chunks: read where it is added)
              float r[32];
              load_row_chunk<32>(r, p.residual, (long long)m * p.ldr, n0, p.N, p.res_dtype, full32);
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] += r[j];
            }
          }
          if (scale != 1.0f) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= scale;
          }
          if (ew == 0 && lane == 0 && b == 0) FL_STAMP(24);
          // ---- ragged row end: a TMA store writes whole 16-byte granules, so the
          // columns past the last full granule are written with plain stores.
          if (!full_chunk && m_ok && n0 < p.n_tma) {
            // every whole 16-byte granule below n_tma (the columns from n_tma on follow below)
            constexpr int EPG = (OUT == DT_F32) ? 4 : 8;  // elements per granule
            char* dst = reinterpret_cast<char*>(p.out) + ((long long)m * p.ldo + n0) * (OUT == DT_F32 ? 4 : 2);
#pragma unroll
            for (int c = 0; c < GPB; ++c) {
              if (n0 + (c + 1) * EPG > p.n_tma) break;
              uint32_t w4[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                if constexpr (OUT == DT_F32) w4[k] = __float_as_uint(v[4 * c + k]);
                else w4[k] = pack2<OUT>(v[8 * c + 2 * k], v[8 * c + 2 * k + 1]);
              }
              asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(dst + 16 * c), "r"(w4[0]), "r"(w4[1]),
                           "r"(w4[2]), "r"(w4[3])
                           : "memory");
            }
          }
          if (n0 + 32 > p.n_tma && n0 < p.N && m_ok) {
            const int j0 = max(p.n_tma - n0, 0);
            const int j1 = min(p.N - n0, 32);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j >= j0 && j < j1) store_elem<OUT>(p.out, (long long)m * p.ldo + n0 + j, v[j]);
          }
          if (tma_chunk) {
            // ---- the block's granules of the 128B-swizzled staging row
#pragma unroll
            for (int c = 0; c < GPB; ++c) {
              uint32_t w4[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                if constexpr (OUT == DT_F32) w4[k] = __float_as_uint(v[4 * c + k]);
                else w4[k] = pack2<OUT>(v[8 * c + 2 * k], v[8 * c + 2 * k + 1]);
              }
              const uint32_t g = (uint32_t)(GPB * hh + c);
              const uint32_t addr = stg + (uint32_t)lane * 128u + ((g ^ (uint32_t)(lane & 7)) << 4);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w4[0]), "r"(w4[1]),
                           "r"(w4[2]), "r"(w4[3])
                           : "memory");
            }
            if (hh == BPC - 1 || b + 1 == nblk) {
              fence_proxy_async_smem();
              __syncwarp();
              if (ew == 0 && lane == 0 && b == BPC - 1) FL_STAMP(26);
              if (lane == 0) {
                tma_store_2d(&tmOut, stg, nc0, row0);
                bulk_commit_group();
                if (ew == 0 && b == BPC - 1) FL_STAMP(20);
                if (ew == 0 && b == 2 * BPC - 1) FL_STAMP(28);
              }
            }
          }
          if (acc_any && b + 1 < nblk) tmem_wait_ld();  // the next block's accumulator has arrived
          if (b + 1 == nblk) {
            // this warp's TMEM reads of the tile are done: hand its share back to the MMA warp
            // (in a pair, to the leader's barrier)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if (PAIR && rank != 0) mbar_arrive_remote(mapa_shared(tempty_bar(buf), 0));
              else mbar_arrive(tempty_bar(buf));
            }
          }
        }
        if (ew == 0 && lane == 0) FL_STAMP(21);
        if (ew == 0 && lane == 0 && local == 0) FL_STAMP(7);
      }
      if (ew == 0 && lane == 0) FL_STAMP(9);
      if (lane == 0) bulk_wait_group<0>();
      if (ew == 0 && lane == 0) FL_STAMP(22);
    } else {
      // ---------------- swap-AB layout: TMEM lane = output column n, TMEM column = output row m.
      // Split-K (S > 1): every CTA publishes its fp32 partial tile in its own shared
      // memory; CTA r then sums the S partials (in rank order) of TMEM lanes
      // [r·128/S, (r+1)·128/S) and finishes those output columns.  Warp ew owns 32
      // of those lanes and a range of rows.  The finishing loop stays rolled (eight
      // independent rows a trip): it runs once per CTA, so its instructions come
      // from L2, and a short body keeps that fetch small.
      const uint32_t red_base = smem_base + p.red_off;
      const int L = 128 / S;
      const int groups = L / 32;
      const int g = (S == 1) ? q : ew % groups;           // S = 1: a warp finishes a lane quarter it may read
      const int parts = kEpiWarps / groups;
      const int part = (S == 1) ? (ew >> 2) : ew / groups;
      const int lrow = (int)rank * L + g * 32 + lane;     // TMEM lane = column within the tile
      const int mcnt = ((p.mma_n + parts - 1) / parts + 7) & ~7;  // rows per warp, a multiple of 8
      const int mb = part * mcnt;
      const int mlen = max(0, min(mcnt, p.mma_n - mb));   // accumulator columns of this warp
      const uint32_t my_row = red_base + (uint32_t)(q * 32 + lane) * p.red_pitch;  // published row
      const uint32_t sum_row = red_base + (uint32_t)lrow * p.red_pitch;            // finished row
      const uint32_t rst = smem_base + p.res_off + (uint32_t)ew * 2u * p.res_blk_bytes;
      const bool res_async = has_res && p.res_async;
      const int res_es = (p.res_dtype == DT_F32) ? 4 : 2;
      constexpr int eo = (OUT == DT_F32) ? 4 : 2;
      Item itm;
      for (; get_item(p, cluster_id, num_clusters, kb_begin, kb_end, (int)local, itm); ++local) {
        int ta, tb;
        tile_coords(itm.tile, p, ta, tb);
        const bool acc_any = itm.kb1 > itm.kb0;
        const uint32_t buf = local & 1u;
        const uint32_t tph = (local >> 1) & 1u;
        const int m_lo = tb * p.mma_n + mb;                 // first output row of this warp
        const int rows = max(0, min(mlen, p.M - m_lo));
        const int n_w0 = ta * 128 + (int)rank * L + g * 32;
        const int n = n_w0 + lane;
        const bool n_ok = n < p.N;
        // the residual's first block travels while the main loop runs
        if (res_async && rows > 0) stage_residual(p, rst, m_lo, min(32, rows), n_w0, lane);
        if (!warp_wait_bounded(tfull_bar(buf), tph, p, lane)) { ok = false; break; }
        tc_fence_after();
        if (ew == 0 && lane == 0) {
          if (local == 0) FL_STAMP(6);
          FL_STAMP(8);
        }
        const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + buf * (uint32_t)p.mma_n;

        if (S > 1) {
          // the two warps of a lane quarter publish alternate 32-column chunks
#pragma unroll 1
          for (int cc = (ew >> 2) * 32; cc < p.mma_n; cc += 64) {
            uint32_t r[32];
            if (acc_any) {
              tmem_ld32(tacc + (uint32_t)cc, r);
              tmem_wait_ld();
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) r[j] = 0u;
            }
#pragma unroll
            for (int c = 0; c < 8; ++c)
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(my_row + (uint32_t)(cc + 4 * c) * 4u),
                           "r"(r[4 * c]), "r"(r[4 * c + 1]), "r"(r[4 * c + 2]), "r"(r[4 * c + 3])
                           : "memory");
          }
          // the copy engine reads these rows: generic writes before async-proxy reads
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          const uint32_t slice_bytes = (uint32_t)L * p.red_pitch;
          const uint32_t recv = red_base + 128u * p.red_pitch;  // S-1 slots of one slice each
          if (lane == 0) {
            mbar_arrive(tempty_bar(buf));
            // expect the peers' slices before telling anyone this CTA is ready for them
            if (ew == 0) mbar_arrive_expect_tx(recv_bar, (uint32_t)(S - 1) * slice_bytes);
            for (int rk = 0; rk < S; ++rk) mbar_arrive_remote(mapa_shared(red_ready_bar, (uint32_t)rk));
          }
          if (!warp_wait_bounded(red_ready_bar, 0, p, lane, true)) ok = false;
          if (ew == 0 && lane == 0) FL_STAMP(12);
          // Every CTA has published and its stages are dead: push slice k of this CTA's
          // partial (rows [k·L, k·L + L), contiguous) into CTA k's receive slot for this
          // rank, with the copy engine.
          if (ok && ew == 0 && lane == 0) {
            for (int k = 0; k < S; ++k) {
              if (k == (int)rank) continue;
              const int slot = ((int)rank < k) ? (int)rank : (int)rank - 1;
              bulk_copy_to_peer(mapa_shared(recv + (uint32_t)slot * slice_bytes, (uint32_t)k),
                                red_base + (uint32_t)(k * L) * p.red_pitch, slice_bytes,
                                mapa_shared(recv_bar, (uint32_t)k));
            }
          }
          // (waited even after a failed wait above: a peer that got through may be
          // writing into this CTA, which must not leave before the bytes land)
          if (!warp_wait_bounded(recv_bar, 0, p, lane, true)) ok = false;
          if (ew == 0 && lane == 0) FL_STAMP(13);
          // tell the sources their copies have landed (they stay resident until then)
          if (ok && ew == 0 && lane == 0)
            for (int k = 0; k < S; ++k)
              if (k != (int)rank) mbar_arrive_remote(mapa_shared(red_done_bar, (uint32_t)k));
          // Sum the S partials of this CTA's slice in rank order (this CTA's own rows and
          // the received slots, all local) and write the sums over the own rows.
          {
            const uint32_t slice = red_base + (uint32_t)(rank * L) * p.red_pitch;
            constexpr uint32_t kStep = kEpiWarps * 32u * 16u;
            if (ok) {
#pragma unroll 1
              for (uint32_t o = (uint32_t)(ew * 32 + lane) * 16u; o < slice_bytes; o += kStep) {
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  if (k >= S) break;
                  const uint32_t a = (k == (int)rank) ? slice + o
                                                      : recv + (uint32_t)(k < (int)rank ? k : k - 1) * slice_bytes + o;
                  const float4 v = ld_shared_f4(a);
                  if (k == 0) {
                    acc = v;
                  } else {
                    acc.x += v.x;
                    acc.y += v.y;
                    acc.z += v.z;
                    acc.w += v.w;
                  }
                }
                st_shared_f4(slice + o, acc);
              }
            }
            // every warp's sums are in place before any warp finishes rows
            asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
            if (ew == 0 && lane == 0) FL_STAMP(14);
          }
        }

        // ---- finish: rows in blocks of 32 (residual blocks double-buffered), eight rows a
        // trip.  Rows past the warp's count are computed from valid (stale) shared memory and
        // never stored.
        float bias_n = 0.0f;
        if (has_bias && p.bias_axis == 0 && n_ok) bias_n = ldg_pinned(p.bias, n, p.bias_dtype);
        const float scale_v = p.scale;
        if (ok) {
#pragma unroll 1
          for (int bm = 0; bm < rows; bm += 32) {
            const int cnt = min(32, rows - bm);
            const uint32_t rcur = rst + (uint32_t)((bm >> 5) & 1) * p.res_blk_bytes;
            if (res_async) {
              if (bm + 32 < rows) {
                stage_residual(p, rst + (uint32_t)(((bm >> 5) + 1) & 1) * p.res_blk_bytes, m_lo + bm + 32,
                               min(32, rows - bm - 32), n_w0, lane);
                cp_async_wait<1>();
              } else {
                cp_async_wait<0>();
              }
              __syncwarp();  // every lane's copies of the block have landed
            }
            // lane l holds the bias of row bm + l (bias along M), read back by shuffle
            float bias_l = 0.0f;
            if (has_bias && p.bias_axis == 1 && lane < cnt) bias_l = ldg_pinned(p.bias, m_lo + bm + lane, p.bias_dtype);
#pragma unroll 1
            for (int j = 0; j < cnt; j += 8) {
              const int mc = mb + bm + j;  // accumulator column of row m_lo + bm + j
              float x[8];
              if (S > 1) {
                const float4 v0 = ld_shared_f4(sum_row + (uint32_t)mc * 4u);
                const float4 v1 = ld_shared_f4(sum_row + (uint32_t)mc * 4u + 16u);
                x[0] = v0.x, x[1] = v0.y, x[2] = v0.z, x[3] = v0.w;
                x[4] = v1.x, x[5] = v1.y, x[6] = v1.z, x[7] = v1.w;
              } else if (acc_any) {
                uint32_t r0[4], r1[4];
                tmem_ld4(tacc + (uint32_t)mc, r0);
                tmem_ld4(tacc + (uint32_t)mc + 4u, r1);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 4; ++i) x[i] = __uint_as_float(r0[i]), x[4 + i] = __uint_as_float(r1[i]);
              } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = 0.0f;
              }
              float rv[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) rv[i] = 0.0f;
              if (res_async) {
                const uint32_t ra = rcur + (uint32_t)(j * 32 + lane) * (uint32_t)res_es;
                if (res_es == 4) {
#pragma unroll
                  for (int i = 0; i < 8; ++i) rv[i] = __uint_as_float(ld_shared_u32(ra + (uint32_t)i * 128u));
                } else if (p.res_dtype == DT_BF16) {
#pragma unroll
                  for (int i = 0; i < 8; ++i) rv[i] = __uint_as_float((uint32_t)ld_shared_u16(ra + (uint32_t)i * 64u) << 16);
                } else {
#pragma unroll
                  for (int i = 0; i < 8; ++i) rv[i] = __half2float(__ushort_as_half(ld_shared_u16(ra + (uint32_t)i * 64u)));
                }
              } else if (has_res && n_ok) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  if (j + i < cnt) rv[i] = ldg_pinned(p.residual, (long long)(m_lo + bm + j + i) * p.ldr + n, p.res_dtype);
              }
              const long long row0 = (long long)(m_lo + bm + j);
              char* orow = reinterpret_cast<char*>(p.out) + (row0 * p.ldo + n) * eo;
              const long long ostep = p.ldo * eo;
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                float xv = x[i];
                if (has_bias) xv += (p.bias_axis == 0) ? bias_n : __shfl_sync(0xffffffffu, bias_l, (j + i) & 31);
                if constexpr (ACT == ACT_GELU) {
                  // GELU_AUX_BIAS: the pre-activation v, in the output type
                  if (has_aux && n_ok && j + i < cnt) store_elem<OUT>(p.aux, (row0 + i) * p.ldo + n, xv);
                }
                if (has_mask) {
                  const uint32_t word = __ballot_sync(0xffffffffu, n_ok && xv > 0.0f);
                  const int wcol = n_w0 >> 5;
                  if (lane == 0 && j + i < cnt && (long long)wcol * 32 < p.N)
                    p.aux[(row0 + i) * p.ld_aux + wcol] = word;
                }
                const float y = (activate<ACT, OUT != DT_F32>(xv, 0.0f) + rv[i]) * scale_v;
                if (n_ok && j + i < cnt) {
                  char* dst = orow + i * ostep;
                  if constexpr (OUT == DT_F32) *reinterpret_cast<float*>(dst) = y;
                  else if constexpr (OUT == DT_BF16) *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(y);
                  else *reinterpret_cast<__half*>(dst) = __float2half_rn(y);
                }
              }
            }
            __syncwarp();  // the block's buffer is refilled two blocks later
          }
        }
        if (ew == 0 && lane == 0) {
          if (local == 0) FL_STAMP(7);
          FL_STAMP(9);
        }
        if (S == 1) {
          // this warp's TMEM reads of the buffer are done
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty_bar(buf));
          continue;
        }
        // nobody leaves while its copies into the peers may still be reading its rows
        if (ew == 0 && !warp_wait_bounded(red_done_bar, 0, p, lane, true)) ok = false;
        break;  // a split-K cluster owns exactly one tile
      }
      cp_async_wait<0>();  // no copy into shared memory outlives the loop
    }
    (void)ok;
    __syncwarp();
  }

  // ================================================================ teardown
  // Every thread of every role arrives here converged, after its last TMEM
  // read, MMA (drained) and copy; only then is TMEM released.
  if (threadIdx.x == 0) FL_STAMP(10);
  __syncthreads();
  // A cluster (CTA pair or split-K group) stays resident until no CTA can still touch
  // another's barriers, shared memory or TMEM: after a bounded wait gave up in one CTA,
  // a peer that got through may still arrive on its barriers or copy into it.  Every
  // wait before this point is bounded, so every CTA of the cluster reaches it.
  if (S > 1 || PAIR) cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, p.tmem_cols);
    else tmem_dealloc(tmem_base, p.tmem_cols);
    if (lane == 0) FL_STAMP(11);
  }
}

}  // namespace fl
