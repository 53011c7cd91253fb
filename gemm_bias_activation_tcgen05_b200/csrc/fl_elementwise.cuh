// fl_elementwise.cuh — HBM-bound kernels of the fused linear layer:
//
//   * fl_relu_backward_kernel: dpre = grad ⊙ bit(mask), the backward use of the
//     RELU_AUX_BIAS mask (cuBLASLt epilog page: the aux ReLU mask serves the
//     backward pass).  A warp per block of 32 mask words of a row.
//   * fl_bwd_bgrad_kernel: the same step, or dpre = grad · GELU'(v) from the
//     pre-activation a GELU_AUX_BIAS forward stored, fused with the bias
//     gradient dbias[n] = Σ_m dpre[m,n] (Linear+GELU page §2.2.1: the backward
//     gradient is fused as well).
//   * fl_ew_step_kernel: ONE epilogue step per launch (bias, activation with
//     optional mask, residual, scale, GeGLU product) over a row-major matrix —
//     the unfused GEMM-then-elementwise design of the Linear+GELU page
//     (zwxr.cn/news/294525, §3.1) and the eager chain of the mHC page
//     (mhpn.cn/news/2504128, §3.4).  It exists only to measure the HBM round
//     trips that the fused kernel removes.
//
// Both are grid-stride loops over 32-element row segments: consecutive threads
// touch consecutive 64/128-byte segments of a row, so each warp reads a
// contiguous 2-4 KB span.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fl_gemm.cuh"

namespace fl {

template <int DT>
struct ElemT;
template <>
struct ElemT<DT_BF16> { using T = __nv_bfloat16; static constexpr uint32_t sign = 0x8000u; };
template <>
struct ElemT<DT_F16> { using T = __half; static constexpr uint32_t sign = 0x8000u; };
template <>
struct ElemT<DT_F32> { using T = float; static constexpr uint32_t sign = 0x80000000u; };

// ---------------------------------------------------------------- backward with bias gradient
enum BwdMode { BWD_DRELU = 0, BWD_DGELU = 1 };

struct BwdParams {
  const void* grad;      // [M, ldg] of DT
  const uint32_t* mask;  // DRELU: [M, words] packed ReLU mask
  const void* v;         // DGELU: [M, ldv] of DT, the stored pre-activation
  void* dpre;            // [M, ldd] of DT
  float* dbias;          // [N] fp32, or null (no bias gradient)
  float* ws;             // row_blocks x ws_ld fp32 column partial sums, one row per row block
  long long M, N, ldg, ldv, ldd, words, ws_ld;
  int rows_per_block, row_blocks, vec_ok;
};

// GELU'(v) = Φ(v) + v·φ(v) in fp32, with erf as in the forward epilogue; the e^(-x²) of
// that erf at x = v/√2 is e^(-v²/2), so φ(v) = e^(-v²/2)/√(2π) needs no second exponential
__device__ __forceinline__ float gelu_erf_grad_f(float v) {
  float e;
  const float Phi = fmaf(0.5f, erf_as_e(v * 0.70710678118654752f, e), 0.5f);
  return fmaf(v * 0.39894228040143268f, e, Phi);
}

// Grid (column groups, row blocks).  A strip is 32 16-byte vectors of a row; warp w of a
// CTA takes strip 8·blockIdx.x + w (lane l its l-th vector) and all eight warps walk the
// same rows of the block, RU rows a trip, so the CTA reads and writes each row as
// 8·512 contiguous bytes (strips of eight different rows per CTA stream a third slower).
// Each thread keeps fp32 partial sums of its VE columns over the block's rows and stores
// them as the block's row of the workspace; fl_bgrad_reduce_kernel then adds the row
// blocks in a fixed order, so the result does not depend on the schedule.
// Three CTAs of 256 threads per SM: the loop's four rows of packed vectors, the
// partial sums and the row pointers fit 85 registers without spills (at four CTAs they spill).
template <int DT, int MODE>
__global__ void __launch_bounds__(256, 3) fl_bwd_bgrad_kernel(const BwdParams P) {
  using T = typename ElemT<DT>::T;
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  constexpr int ESZ = sizeof(T);
  constexpr int VE = 16 / ESZ;  // elements per 16-byte vector
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long strip0 = ((long long)blockIdx.x * 8 + warp) * 32 * VE;  // first column of the strip
  if (strip0 >= P.N) return;  // a strip past the last column (no CTA-wide barrier below)
  const int rb = blockIdx.y;
  const long long c0 = strip0 + (long long)lane * VE;
  const long long r0 = (long long)rb * P.rows_per_block;
  const long long r1 = min(P.M, r0 + P.rows_per_block);
  const bool any = c0 < P.N;
  const bool vec = P.vec_ok && c0 + VE <= P.N;
  const T* grad = reinterpret_cast<const T*>(P.grad);
  const T* vv = reinterpret_cast<const T*>(P.v);
  T* dpre = reinterpret_cast<T*>(P.dpre);
  float part[VE];
#pragma unroll
  for (int i = 0; i < VE; ++i) part[i] = 0.0f;
  // four rows a trip: every load of the trip is in flight before the first use; the
  // vectors stay packed until then.  Row pointers advance by the pitch (no per-row
  // 64-bit index products in the loop).
  constexpr int RU = 4;
  const char* gp = reinterpret_cast<const char*>(grad + r0 * P.ldg + c0);
  const char* vp = reinterpret_cast<const char*>(vv + (MODE == BWD_DGELU ? r0 * P.ldv + c0 : 0));
  char* dp = reinterpret_cast<char*>(dpre + r0 * P.ldd + c0);
  const uint32_t* mp = P.mask + (MODE == BWD_DRELU ? r0 * P.words + (c0 >> 5) : 0);
  const long long gs = P.ldg * ESZ, vs = P.ldv * ESZ, ds = P.ldd * ESZ;
  const int sh = (int)(c0 & 31);
  for (long long mb = r0; mb < r1 && any; mb += RU) {
    const int nrow = (int)min((long long)RU, r1 - mb);
    uint4 gq[RU], vq[RU];
    uint32_t word[RU];
#pragma unroll
    for (int u = 0; u < RU; ++u) {
      gq[u] = make_uint4(0u, 0u, 0u, 0u);
      vq[u] = make_uint4(0u, 0u, 0u, 0u);
      word[u] = 0u;
      if (u >= nrow) continue;
      if (vec) {
        gq[u] = __ldg(reinterpret_cast<const uint4*>(gp + u * gs));
        if (MODE == BWD_DGELU) vq[u] = __ldg(reinterpret_cast<const uint4*>(vp + u * vs));
      } else {
        T* ge = reinterpret_cast<T*>(&gq[u]);
        T* ve = reinterpret_cast<T*>(&vq[u]);
#pragma unroll
        for (int i = 0; i < VE; ++i) {
          if (c0 + i < P.N) {
            ge[i] = reinterpret_cast<const T*>(gp + u * gs)[i];
            if (MODE == BWD_DGELU) ve[i] = reinterpret_cast<const T*>(vp + u * vs)[i];
          }
        }
      }
      // the VE columns lie in one mask word (VE divides 32)
      if (MODE == BWD_DRELU) word[u] = __ldg(mp + u * P.words);
    }
#pragma unroll
    for (int u = 0; u < RU; ++u) {
      if (u >= nrow) continue;
      const T* ge = reinterpret_cast<const T*>(&gq[u]);
      const T* ve = reinterpret_cast<const T*>(&vq[u]);
      float d[VE];
#pragma unroll
      for (int i = 0; i < VE; ++i) {
        const float gi = static_cast<float>(ge[i]);
        if (MODE == BWD_DRELU) d[i] = ((word[u] >> (sh + i)) & 1u) ? gi : gi * 0.0f;  // keeps grad's sign
        else d[i] = gi * gelu_erf_grad_f(static_cast<float>(ve[i]));
      }
      T* de = reinterpret_cast<T*>(dp + u * ds);
      if (vec) {
        uint4 q;
        T* e = reinterpret_cast<T*>(&q);
#pragma unroll
        for (int i = 0; i < VE; ++i) e[i] = static_cast<T>(d[i]);
        *reinterpret_cast<uint4*>(de) = q;
      } else {
#pragma unroll
        for (int i = 0; i < VE; ++i)
          if (c0 + i < P.N) de[i] = static_cast<T>(d[i]);
      }
#pragma unroll
      for (int i = 0; i < VE; ++i) part[i] += d[i];
    }
    gp += RU * gs;
    if (MODE == BWD_DGELU) vp += RU * vs;
    dp += RU * ds;
    if (MODE == BWD_DRELU) mp += RU * P.words;
  }
  if (P.dbias == nullptr || !any) return;
  float* dst = P.ws + (long long)rb * P.ws_ld + c0;
  if (c0 + VE <= P.N) {  // (ws rows and c0 are 16-byte aligned)
#pragma unroll
    for (int i = 0; i < VE; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(part[i], part[i + 1], part[i + 2], part[i + 3]);
  } else {
#pragma unroll
    for (int i = 0; i < VE; ++i)
      if (c0 + i < P.N) dst[i] = part[i];
  }
}

// dbias[c] = Σ over the row blocks of ws[rb][c].  A CTA of 32 x 32 threads takes 32
// columns; thread (g, l) adds row blocks g, g + 32, g + 64, ... of column l in ascending
// order (all its loads in flight at once for up to 512 row blocks), then thread (0, l)
// adds the 32 group sums in group order: a fixed order, whatever the schedule.
// Launched after fl_bwd_bgrad_kernel with programmatic dependent launch; the wait
// below covers that kernel's stores.
__global__ void __launch_bounds__(1024, 1) fl_bgrad_reduce_kernel(const float* __restrict__ ws, float* dbias,
                                                                  long long N, long long ws_ld, int row_blocks) {
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  const int g = threadIdx.x >> 5, l = threadIdx.x & 31;
  const long long c = (long long)blockIdx.x * 32 + l;
  __shared__ float red[32][33];
  float s = 0.0f;
  if (c < N) {
    for (int b0 = g; b0 < row_blocks; b0 += 32 * 16) {
      float t[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int b = b0 + 32 * k;
        t[k] = b < row_blocks ? __ldcg(ws + (long long)b * ws_ld + c) : 0.0f;
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) s += t[k];
    }
  }
  red[g][l] = s;
  __syncthreads();
  if (g == 0 && c < N) {
    float r = red[0][l];
#pragma unroll
    for (int k = 1; k < 32; ++k) r += red[k][l];
    dbias[c] = r;
  }
}

// ---------------------------------------------------------------- LayerNorm after the tail
struct LnParams {
  const void* x;      // [M, ldx] of XT
  const void* gamma;  // [N] of param_dtype, or null (1)
  const void* beta;   // [N] of param_dtype, or null (0)
  void* z;            // [M, ldz] of ZT (may be x itself, with ldz == ldx)
  long long M, N, ldx, ldz;
  int param_dtype, vec_ok;
  int pvec;  // gamma/beta 16-byte aligned: loaded as vectors
  int zvec;  // z base and pitch allow vector stores of a thread's VE outputs
  float eps;
};

// VE consecutive parameters from c0 (16-byte vector loads), or `dflt` for a null pointer
template <int VE>
__device__ __forceinline__ void load_params_vec(const void* p, long long c0, int dt, float dflt, float (&o)[VE]) {
  if (p == nullptr) {
#pragma unroll
    for (int i = 0; i < VE; ++i) o[i] = dflt;
    return;
  }
  if (dt == DT_F32) {
#pragma unroll
    for (int j = 0; j < VE / 4; ++j) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + c0) + j);
      o[4 * j] = f.x, o[4 * j + 1] = f.y, o[4 * j + 2] = f.z, o[4 * j + 3] = f.w;
    }
  } else {
    // 16-bit parameters: VE = 4 reads 8 bytes, VE = 8 reads 16 bytes
    uint32_t w[VE / 2];
    if constexpr (VE == 8) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p) + c0));
      w[0] = q.x, w[1] = q.y, w[2] = q.z, w[3] = q.w;
    } else {
      const uint2 q = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(p) + c0));
      w[0] = q.x, w[1] = q.y;
    }
#pragma unroll
    for (int i = 0; i < VE; ++i) {
      const uint16_t h = (uint16_t)(w[i >> 1] >> (16 * (i & 1)));
      o[i] = (dt == DT_BF16) ? __uint_as_float((uint32_t)h << 16) : __half2float(__ushort_as_half(h));
    }
  }
}

// Sum of one value per thread over the NW warps of the CTA, in a fixed order (butterfly
// in each warp, then the warp sums in warp order).
template <int NW>
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red is free (a previous call has been read)
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = red[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) s += red[w];
  return s;
}

// z = (x − μ)·rstd·γ + β over each row (mHC page §3.2: the mean and variance of the
// row, then the normalisation, in one kernel: one read and one write of the row).
// A CTA of TPB threads normalises rows blockIdx.x, blockIdx.x + gridDim.x, ... (one
// resident wave).  A row of up to TPB·VMAX 16-byte vectors stays in registers across
// the three steps (mean, Σ(x − μ)², normalise).  When rows are 16-byte aligned, each
// thread copies its vectors of the CTA's NEXT row into shared memory (cp.async) as
// soon as it has taken the current row into registers, so that row's read runs while
// this one is reduced and stored; each thread reads back only the slots it copied.
// A longer row is read again for the later steps.  Rows of up to 4096 elements take
// 128-thread CTAs keeping 32 elements a thread; longer rows take 256 threads.
template <int XT, int ZT, int TPB>
__global__ void __launch_bounds__(TPB, TPB == 128 ? 6 : 3) fl_layernorm_kernel(const LnParams P) {
  using TX = typename ElemT<XT>::T;
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  constexpr int VE = 16 / sizeof(TX);             // elements per 16-byte vector of x
  constexpr int VMAX = TPB == 128 ? 32 / VE : 4;  // vectors a thread keeps in registers
  constexpr int NW = TPB / 32;
  __shared__ float red[NW];
  __shared__ __align__(16) uint4 stage[VMAX * TPB];  // the next row, slot k·TPB + t for thread t
  const long long N = P.N;
  const int t = threadIdx.x;
  const bool in_regs = N <= (long long)TPB * VMAX * VE;
  const bool pipelined = in_regs && P.vec_ok;
  const uint32_t stage_base = (uint32_t)__cvta_generic_to_shared(stage);
  auto row_ptr = [&](long long m) { return reinterpret_cast<const TX*>(P.x) + m * P.ldx; };
  // copy this thread's whole vectors of row m into its stage slots
  auto prefetch = [&](long long m) {
    const TX* x = row_ptr(m);
#pragma unroll
    for (int k = 0; k < VMAX; ++k) {
      const long long c0 = ((long long)k * TPB + t) * VE;
      if (c0 + VE <= N) cp_async_16(stage_base + (uint32_t)(k * TPB + t) * 16u, x + c0, 16u);
    }
    cp_async_commit();
  };
  if (pipelined && blockIdx.x < P.M) prefetch(blockIdx.x);
  for (long long m = blockIdx.x; m < P.M; m += gridDim.x) {
    const TX* x = row_ptr(m);
    auto load_vec = [&](long long c0, float (&v)[VE]) {
      if (P.vec_ok && c0 + VE <= N) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(x + c0));
        const TX* e = reinterpret_cast<const TX*>(&q);
#pragma unroll
        for (int i = 0; i < VE; ++i) v[i] = static_cast<float>(e[i]);
      } else {
#pragma unroll
        for (int i = 0; i < VE; ++i) v[i] = (c0 + i < N) ? static_cast<float>(x[c0 + i]) : 0.0f;
      }
    };
    float xv[VMAX][VE];
    float s = 0.0f;
    if (pipelined) {
      cp_async_wait<0>();  // this thread's copies of row m have landed
#pragma unroll
      for (int k = 0; k < VMAX; ++k) {
        const long long c0 = ((long long)k * TPB + t) * VE;
#pragma unroll
        for (int i = 0; i < VE; ++i) xv[k][i] = 0.0f;
        if (c0 + VE <= N) {
          const uint4 q = *reinterpret_cast<const uint4*>(&stage[k * TPB + t]);
          const TX* e = reinterpret_cast<const TX*>(&q);
#pragma unroll
          for (int i = 0; i < VE; ++i) xv[k][i] = static_cast<float>(e[i]);
        } else if (c0 < N) {
          load_vec(c0, xv[k]);  // the row's partial last vector
        }
      }
#pragma unroll
      for (int k = 0; k < VMAX; ++k)
#pragma unroll
        for (int i = 0; i < VE; ++i) s += xv[k][i];
      // the slots are free once their values have been used (the sum above)
      if (m + gridDim.x < P.M) prefetch(m + gridDim.x);
    } else if (in_regs) {
      // every load of the row is issued before the first use, so their latencies overlap
#pragma unroll
      for (int k = 0; k < VMAX; ++k) {
        const long long c0 = ((long long)k * TPB + t) * VE;
#pragma unroll
        for (int i = 0; i < VE; ++i) xv[k][i] = 0.0f;
        if (c0 < N) load_vec(c0, xv[k]);
      }
#pragma unroll
      for (int k = 0; k < VMAX; ++k)
#pragma unroll
        for (int i = 0; i < VE; ++i) s += xv[k][i];
    } else {
      for (long long c0 = (long long)t * VE; c0 < N; c0 += (long long)TPB * VE) {
        float v[VE];
        load_vec(c0, v);
#pragma unroll
        for (int i = 0; i < VE; ++i) s += v[i];
      }
    }
    const float mean = block_sum<NW>(s, red) / (float)N;
    float q = 0.0f;
    if (in_regs) {
#pragma unroll
      for (int k = 0; k < VMAX; ++k) {
        const long long c0 = ((long long)k * TPB + t) * VE;
#pragma unroll
        for (int i = 0; i < VE; ++i)
          if (c0 + i < N) q += (xv[k][i] - mean) * (xv[k][i] - mean);
      }
    } else {
      for (long long c0 = (long long)t * VE; c0 < N; c0 += (long long)TPB * VE) {
        float v[VE];
        load_vec(c0, v);
#pragma unroll
        for (int i = 0; i < VE; ++i)
          if (c0 + i < N) q += (v[i] - mean) * (v[i] - mean);
      }
    }
    const float var = block_sum<NW>(q, red) / (float)N;
    const float rstd = 1.0f / sqrtf(var + P.eps);
    auto finish = [&](long long c0, const float (&v)[VE]) {
      if (c0 + VE <= N && P.pvec && P.zvec) {
        // whole vector: parameters by 16-byte loads, the VE outputs by one or two vector stores
        float g[VE], b[VE], o[VE];
        load_params_vec<VE>(P.gamma, c0, P.param_dtype, 1.0f, g);
        load_params_vec<VE>(P.beta, c0, P.param_dtype, 0.0f, b);
#pragma unroll
        for (int i = 0; i < VE; ++i) o[i] = (v[i] - mean) * rstd * g[i] + b[i];
        char* dst = reinterpret_cast<char*>(P.z) + (m * P.ldz + c0) * (ZT == DT_F32 ? 4 : 2);
        if constexpr (ZT == DT_F32) {
#pragma unroll
          for (int j = 0; j < VE / 4; ++j)
            reinterpret_cast<float4*>(dst)[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
        } else {
          uint32_t w[VE / 2];
#pragma unroll
          for (int j = 0; j < VE / 2; ++j) w[j] = pack2<ZT>(o[2 * j], o[2 * j + 1]);
          if constexpr (VE == 8) *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
          else *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
        }
        return;
      }
#pragma unroll
      for (int i = 0; i < VE; ++i) {
        const long long c = c0 + i;
        if (c < N) {
          const float g = P.gamma ? load_elem(P.gamma, c, P.param_dtype) : 1.0f;
          const float b = P.beta ? load_elem(P.beta, c, P.param_dtype) : 0.0f;
          store_elem<ZT>(P.z, m * P.ldz + c, (v[i] - mean) * rstd * g + b);
        }
      }
    };
    if (in_regs) {
#pragma unroll
      for (int k = 0; k < VMAX; ++k) {
        const long long c0 = ((long long)k * TPB + t) * VE;
        if (c0 < N) finish(c0, xv[k]);
      }
    } else {
      for (long long c0 = (long long)t * VE; c0 < N; c0 += (long long)TPB * VE) {
        float v[VE];
        load_vec(c0, v);
        finish(c0, v);
      }
    }
  }
  cp_async_wait<0>();  // no copy of this CTA is still in flight when it exits
}

// The same normalisation for the common layout: x, z and the parameters 16-byte aligned
// with 16-byte row pitches, N a multiple of the vector width and at most TPB·VMAX
// vectors.  Column offsets are 32-bit, the validity of each of a thread's vectors is
// fixed for the whole launch, and every access is a whole vector, which keeps the
// instruction count per element small.  Each thread keeps its vectors of the CTA's next
// LN_DEPTH rows in flight (one cp.async group per row, in LN_DEPTH shared-memory slots).
// (Two rows deep measured slower on 2048 x 4096 fp32: 15.7 vs 13.4 us; the second slot
// doubles the shared memory of a CTA.)
constexpr int LN_DEPTH = 1;  // rows a CTA of the vector LayerNorm keeps in flight
template <int XT, int ZT, int TPB>
__global__ void __launch_bounds__(TPB, TPB == 128 ? 6 : 4) fl_layernorm_vec_kernel(const LnParams P) {
  using TX = typename ElemT<XT>::T;
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  constexpr int VE = 16 / sizeof(TX);
  constexpr int VMAX = TPB == 128 ? 32 / VE : 4;
  constexpr int NW = TPB / 32;
  constexpr int EZ = (ZT == DT_F32) ? 4 : 2;
  __shared__ float red[NW];
  __shared__ __align__(16) uint4 stage[LN_DEPTH][VMAX * TPB];
  const int t = threadIdx.x;
  const int nvec = (int)(P.N / VE);
  const float inv_n = 1.0f / (float)P.N;
  const uint32_t stage_base = (uint32_t)__cvta_generic_to_shared(stage);
  // copy this thread's vectors of row m into slot `slot` (the caller commits the group)
  auto prefetch = [&](long long m, int slot) {
    const uint4* x = reinterpret_cast<const uint4*>(reinterpret_cast<const TX*>(P.x) + m * P.ldx);
#pragma unroll
    for (int k = 0; k < VMAX; ++k)
      if (k * TPB + t < nvec)
        cp_async_16(stage_base + (uint32_t)((slot * VMAX + k) * TPB + t) * 16u, x + k * TPB + t, 16u);
  };
  // one group per row slot, empty past the last row, so that at the row of iteration i
  // exactly LN_DEPTH - 1 younger groups exist
#pragma unroll
  for (int d = 0; d < LN_DEPTH; ++d) {
    const long long m = blockIdx.x + (long long)d * gridDim.x;
    if (m < P.M) prefetch(m, d);
    cp_async_commit();
  }
  int slot = 0;
  for (long long m = blockIdx.x; m < P.M; m += gridDim.x) {
    float xv[VMAX][VE];
    cp_async_wait<LN_DEPTH - 1>();  // this row's group has landed
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < VMAX; ++k) {
      if (k * TPB + t < nvec) {
        const uint4 q = stage[slot][k * TPB + t];
        const TX* e = reinterpret_cast<const TX*>(&q);
#pragma unroll
        for (int i = 0; i < VE; ++i) xv[k][i] = static_cast<float>(e[i]);
      } else {
#pragma unroll
        for (int i = 0; i < VE; ++i) xv[k][i] = 0.0f;
      }
#pragma unroll
      for (int i = 0; i < VE; ++i) s += xv[k][i];
    }
    // the slot's values are used above: refill it with the row LN_DEPTH rows ahead
    const long long mn = m + (long long)LN_DEPTH * gridDim.x;
    if (mn < P.M) prefetch(mn, slot);
    cp_async_commit();
    slot = (slot + 1 == LN_DEPTH) ? 0 : slot + 1;
    const float mean = block_sum<NW>(s, red) * inv_n;
    float q = 0.0f;
#pragma unroll
    for (int k = 0; k < VMAX; ++k) {
      if (k * TPB + t < nvec) {
#pragma unroll
        for (int i = 0; i < VE; ++i) q += (xv[k][i] - mean) * (xv[k][i] - mean);
      }
    }
    const float rstd = 1.0f / sqrtf(block_sum<NW>(q, red) * inv_n + P.eps);
    char* zrow = reinterpret_cast<char*>(P.z) + m * P.ldz * EZ;
#pragma unroll
    for (int k = 0; k < VMAX; ++k) {
      const int v = k * TPB + t;
      if (v >= nvec) continue;
      float g[VE], b[VE], o[VE];
      load_params_vec<VE>(P.gamma, (long long)v * VE, P.param_dtype, 1.0f, g);
      load_params_vec<VE>(P.beta, (long long)v * VE, P.param_dtype, 0.0f, b);
#pragma unroll
      for (int i = 0; i < VE; ++i) o[i] = (xv[k][i] - mean) * rstd * g[i] + b[i];
      char* dst = zrow + (size_t)v * VE * EZ;
      if constexpr (ZT == DT_F32) {
#pragma unroll
        for (int j = 0; j < VE / 4; ++j)
          reinterpret_cast<float4*>(dst)[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
      } else {
        uint32_t w[VE / 2];
#pragma unroll
        for (int j = 0; j < VE / 2; ++j) w[j] = pack2<ZT>(o[2 * j], o[2 * j + 1]);
        if constexpr (VE == 8) *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        else *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
      }
    }
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------- dReLU
template <int DT>
__global__ void __launch_bounds__(256, 4) fl_relu_backward_kernel(const void* __restrict__ grad_,
                                                               const uint32_t* __restrict__ aux,
                                                               void* __restrict__ dpre_, long long M,
                                                               long long N, long long ldg,
                                                               long long ldd, long long words,
                                                               int vec_ok) {
  using T = typename ElemT<DT>::T;
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  constexpr int ESZ = sizeof(T);
  constexpr int PER16 = 16 / ESZ;             // elements per 16-byte vector
  constexpr int V = 32 * 32 / PER16 / 32;     // vectors per lane in a block of 32 words
  constexpr int U = (ESZ == 2) ? 2 : 1;       // blocks a trip (16-bit: 8 vectors a lane in flight)
  const T* grad = reinterpret_cast<const T*>(grad_);
  T* dpre = reinterpret_cast<T*>(dpre_);
  const int lane = threadIdx.x & 31;
  // A warp takes blocks of 32 mask words (32·32 elements) of one row, U blocks a trip.
  // In a full block lane l moves 16-byte vectors l, l+32, ... of the block, so every
  // warp-wide access is 512 contiguous bytes, and reads its mask bits from the block's
  // 32 words (one coalesced load) by shuffle.  Every load of a trip (mask words and
  // gradient vectors) is issued before the first use.
  const long long wblocks = (words + 31) / 32;
  const long long total = M * wblocks;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long blk0 = warp0; blk0 < total; blk0 += U * nwarps) {
    uint32_t myword[U];
    uint4 x[U][V];
    bool full[U];
    long long base_g[U], base_d[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const long long blk = blk0 + j * nwarps;
      full[j] = false;
      myword[j] = 0u;
      base_g[j] = base_d[j] = 0;
      if (blk >= total) continue;
      const long long m = blk / wblocks;
      const long long w0 = (blk - m * wblocks) * 32;
      base_g[j] = m * ldg + w0 * 32;
      base_d[j] = m * ldd + w0 * 32;
      if (w0 + lane < words) myword[j] = __ldg(aux + m * words + w0 + lane);
      full[j] = vec_ok && w0 + 32 <= words && (w0 + 32) * 32 <= N;
      if (full[j]) {
#pragma unroll
        for (int v = 0; v < V; ++v) x[j][v] = __ldg(reinterpret_cast<const uint4*>(grad + base_g[j]) + v * 32 + lane);
      }
    }
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const long long blk = blk0 + j * nwarps;
      if (blk >= total) continue;
      const T* g = grad + base_g[j];
      T* d = dpre + base_d[j];
      if (full[j]) {
#pragma unroll
        for (int v = 0; v < V; ++v) {
          const int e0 = (v * 32 + lane) * PER16;  // first element of this lane's vector
          const uint32_t bits = __shfl_sync(0xffffffffu, myword[j], e0 >> 5);
          uint32_t* xw = reinterpret_cast<uint32_t*>(&x[j][v]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if constexpr (ESZ == 2) {
              const int b = (e0 & 31) + e * 2;
              // grad·0 keeps the sign of grad (IEEE): clear all but the sign bit
              const uint32_t lo_keep = ((bits >> b) & 1u) ? 0x0000FFFFu : 0x00008000u;
              const uint32_t hi_keep = ((bits >> (b + 1)) & 1u) ? 0xFFFF0000u : 0x80000000u;
              xw[e] &= (lo_keep | hi_keep);
            } else {
              const int b = (e0 & 31) + e;
              xw[e] &= ((bits >> b) & 1u) ? 0xFFFFFFFFu : 0x80000000u;
            }
          }
          reinterpret_cast<uint4*>(d)[v * 32 + lane] = x[j][v];
        }
      } else {
        // ragged block: lane l finishes word w0 + l element by element
        const long long w = (blk - (blk / wblocks) * wblocks) * 32 + lane;
        if (w < words) {
          const long long n0 = w * 32;
          for (int b = 0; b < 32 && n0 + b < N; ++b) {
            T xe = g[lane * 32 + b];
            if (!((myword[j] >> b) & 1u)) {
              if constexpr (ESZ == 2) {
                unsigned short h = *reinterpret_cast<unsigned short*>(&xe);
                h &= 0x8000u;
                xe = *reinterpret_cast<T*>(&h);
              } else {
                uint32_t h = __float_as_uint(xe) & 0x80000000u;
                xe = __uint_as_float(h);
              }
            }
            d[lane * 32 + b] = xe;
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------- unfused steps
enum EwOp : int {
  EW_BIAS_N = 0,   // y[m,n] = x[m,n] + bias[n]
  EW_BIAS_M = 1,   // y[m,n] = x[m,n] + bias[m]
  EW_RELU = 2,     // y = max(x,0); optional mask of x > 0
  EW_GELU = 3,     // exact GELU
  EW_GELU_TANH = 4,
  EW_RESIDUAL = 5, // y = x + r[m,n]
  EW_SCALE = 6,    // y = x * s
  EW_GEGLU_MUL = 7, // y[m,n] = gelu_tanh(x[m,n]) * u[m,n]  (u = operand)
  EW_GELU_SIGMOID = 8
};

struct EwParams {
  const void* src;
  long long lds;
  void* dst;
  long long ldd;
  long long M, N;
  int op;
  const void* operand;  // bias / residual / u
  int operand_dtype;
  long long ldop;
  float scale;
  uint32_t* aux;
  long long ld_aux;
  // element counts of every buffer: an access outside them is skipped and
  // recorded in *err (code 100 + op) instead of being performed
  long long src_elems, dst_elems, op_elems, aux_elems;
  int* err;
};

__device__ __forceinline__ bool ew_in(long long i, long long n, int* err, int code) {
  if (i >= 0 && i < n) return true;
  atomicCAS(err, 0, code);
  return false;
}

template <int DT>
__device__ __forceinline__ float ew_ld(const void* p, long long i) {
  using T = typename ElemT<DT>::T;
  if constexpr (DT == DT_F32) return reinterpret_cast<const float*>(p)[i];
  else if constexpr (DT == DT_BF16) return __bfloat162float(reinterpret_cast<const T*>(p)[i]);
  else return __half2float(reinterpret_cast<const T*>(p)[i]);
}
template <int DT>
__device__ __forceinline__ void ew_st(void* p, long long i, float v) {
  store_elem<DT>(p, i, v);
}

// VE values of type dt from base[i0 ...] widened to fp32: 16- or 8-byte vector loads when
// `vec` (the first element's address is aligned to the vector) and the vector is whole,
// else element by element up to cnt (the rest 0).
template <int VE>
__device__ __forceinline__ void ew_ld_vals(float (&o)[VE], const void* base, long long i0, int dt, int cnt,
                                           bool vec) {
  if (vec && cnt == VE) {
    if (dt == DT_F32) {
      const float4* s = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + i0);
#pragma unroll
      for (int j = 0; j < VE / 4; ++j) {
        const float4 f = __ldg(s + j);
        o[4 * j] = f.x, o[4 * j + 1] = f.y, o[4 * j + 2] = f.z, o[4 * j + 3] = f.w;
      }
    } else {
      uint32_t w[VE / 2];
      const uint16_t* s = reinterpret_cast<const uint16_t*>(base) + i0;
      if constexpr (VE == 8) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(s));
        w[0] = q.x, w[1] = q.y, w[2] = q.z, w[3] = q.w;
      } else {
        const uint2 q = __ldg(reinterpret_cast<const uint2*>(s));
        w[0] = q.x, w[1] = q.y;
      }
#pragma unroll
      for (int j = 0; j < VE; ++j) {
        const uint16_t h = (uint16_t)(w[j >> 1] >> (16 * (j & 1)));
        o[j] = (dt == DT_BF16) ? __uint_as_float((uint32_t)h << 16) : __half2float(__ushort_as_half(h));
      }
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < VE; ++j) {
    o[j] = 0.0f;
    if (j < cnt) o[j] = ldg_pinned(base, i0 + j, dt);
  }
}

// One epilogue step over 16-byte vectors: thread i of the grid-stride sweep takes
// vector v of row m, i = m·nvp + v, where a row has nvp = words·(32/VE) vector slots
// (VE elements of DT per 16 bytes; the slots past N are idle).  Consecutive lanes read
// and write consecutive 16 bytes of a row, and the 32/VE lanes of one mask word are
// aligned lanes of one warp, so the word is formed by shuffles and stored by its first
// lane.  Requires src and dst rows 16-byte aligned (base and pitch); the operands are
// read by vectors when aligned, else element by element.  Every access is checked
// against its buffer's element count (code 100 + op recorded, access skipped).
template <int DT>
__global__ void __launch_bounds__(256) fl_ew_step_vec_kernel(const EwParams P) {
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  using T = typename ElemT<DT>::T;
  constexpr int ES = sizeof(T);
  constexpr int VE = 16 / ES;
  constexpr int VPW = 32 / VE;  // vectors per 32-column mask word
  const int lane = threadIdx.x & 31;
  const long long words = (P.N + 31) / 32;
  const long long nvp = words * VPW;
  const long long total = P.M * nvp;
  const int code = 100 + P.op;
  const int oes = (P.operand_dtype == DT_F32) ? 4 : 2;
  // operand vectors: the base aligned to the vector's bytes, and (for a matrix) the pitch too
  const uint32_t ovec_bytes = (uint32_t)(VE * oes);
  const uint32_t oalign = ovec_bytes >= 16 ? 16u : ovec_bytes;
  const bool op_vec = P.operand != nullptr && (reinterpret_cast<uintptr_t>(P.operand) % oalign) == 0 &&
                      ((P.op != EW_RESIDUAL && P.op != EW_GEGLU_MUL) || ((P.ldop * oes) % oalign) == 0);
  const long long stride = (long long)gridDim.x * blockDim.x;
  // the trip count is warp-uniform (i - lane is the warp's first slot), so every lane of a
  // warp runs the shuffles of a trip
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i - lane < total; i += stride) {
    const bool live = i < total;
    const long long m = live ? i / nvp : 0;
    const long long v = live ? i - m * nvp : 0;
    const long long n0 = v * VE;
    const int cnt = live ? (int)max(0LL, min((long long)VE, P.N - n0)) : 0;
    uint32_t bits = 0u;
    if (cnt > 0) {
      const long long is = m * P.lds + n0;
      const long long id = m * P.ldd + n0;
      bool ok = ew_in(is, P.src_elems, P.err, code) && ew_in(is + cnt - 1, P.src_elems, P.err, code) &&
                ew_in(id, P.dst_elems, P.err, code) && ew_in(id + cnt - 1, P.dst_elems, P.err, code);
      long long io = -1;
      if (P.op == EW_BIAS_N) io = n0;
      else if (P.op == EW_RESIDUAL || P.op == EW_GEGLU_MUL) io = m * P.ldop + n0;
      if (ok && io >= 0)
        ok = ew_in(io, P.op_elems, P.err, code) && ew_in(io + cnt - 1, P.op_elems, P.err, code);
      if (ok && P.op == EW_BIAS_M) ok = ew_in(m, P.op_elems, P.err, code);
      if (ok) {
        float x[VE], opv[VE], y[VE];
        ew_ld_vals<VE>(x, P.src, is, DT, cnt, true);
        if (io >= 0) {
          ew_ld_vals<VE>(opv, P.operand, io, P.operand_dtype, cnt, op_vec);
        } else if (P.op == EW_BIAS_M) {
          const float b = ldg_pinned(P.operand, m, P.operand_dtype);
#pragma unroll
          for (int j = 0; j < VE; ++j) opv[j] = b;
        } else {
#pragma unroll
          for (int j = 0; j < VE; ++j) opv[j] = 0.0f;
        }
#pragma unroll
        for (int j = 0; j < VE; ++j) {
          switch (P.op) {
            case EW_BIAS_N:
            case EW_BIAS_M:
            case EW_RESIDUAL: y[j] = x[j] + opv[j]; break;
            case EW_RELU:
              y[j] = fmaxf(x[j], 0.0f);
              if (x[j] > 0.0f && j < cnt) bits |= 1u << j;
              break;
            case EW_GELU: y[j] = gelu_erf_f(x[j]); break;
            case EW_GELU_TANH: y[j] = gelu_tanh_f<DT != DT_F32>(x[j]); break;
            case EW_GELU_SIGMOID: y[j] = gelu_sigmoid_f(x[j]); break;
            case EW_SCALE: y[j] = x[j] * P.scale; break;
            default: y[j] = gelu_tanh_f<DT != DT_F32>(x[j]) * opv[j]; break;
          }
        }
        if (cnt == VE) {
          uint32_t w[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if constexpr (DT == DT_F32) w[k] = __float_as_uint(y[k]);
            else w[k] = pack2<DT>(y[2 * k], y[2 * k + 1]);
          }
          *reinterpret_cast<uint4*>(reinterpret_cast<T*>(P.dst) + id) = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
#pragma unroll
          for (int j = 0; j < VE; ++j)
            if (j < cnt) store_elem<DT>(P.dst, id + j, y[j]);
        }
      }
    }
    if (P.op == EW_RELU && P.aux != nullptr) {
      // the word's VPW lanes are aligned within the warp (nvp and 32 are multiples of VPW)
      uint32_t word = bits << ((int)(v % VPW) * VE);
#pragma unroll
      for (int o = 1; o < VPW; o <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, o);
      if (live && (v % VPW) == 0) {
        const long long ia = m * P.ld_aux + v / VPW;
        if (ew_in(ia, P.aux_elems, P.err, code)) P.aux[ia] = word;
      }
    }
  }
}

// Storage dtype DT for src/dst (the eager tensors); operands use their own dtype.
// Element-by-element form, for rows that are not 16-byte aligned.
template <int DT>
__global__ void __launch_bounds__(256) fl_ew_step_kernel(const EwParams P) {
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  const long long words = (P.N + 31) / 32;
  const long long total = P.M * words;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long m = i / words;
    const long long w = i - m * words;
    const long long n0 = w * 32;
    uint32_t mask = 0;
    const int cnt = (int)min(32LL, P.N - n0);
    const int code = 100 + P.op;
    for (int j = 0; j < cnt; ++j) {
      const long long n = n0 + j;
      const long long is = m * P.lds + n;
      if (!ew_in(is, P.src_elems, P.err, code)) continue;
      const float x = ew_ld<DT>(P.src, is);
      float y;
      long long io = -1;
      switch (P.op) {
        case EW_BIAS_N: io = n; break;
        case EW_BIAS_M: io = m; break;
        case EW_RESIDUAL:
        case EW_GEGLU_MUL: io = m * P.ldop + n; break;
        default: break;
      }
      if (io >= 0 && !ew_in(io, P.op_elems, P.err, code)) continue;
      // the operand load sits in its own branch (never folded into a select that
      // would issue it for an op that has no operand)
      float opv = 0.0f;
      if (io >= 0) opv = ldg_pinned(P.operand, io, P.operand_dtype);
      switch (P.op) {
        case EW_BIAS_N:
        case EW_BIAS_M: y = x + opv; break;
        case EW_RELU:
          y = fmaxf(x, 0.0f);
          if (x > 0.0f) mask |= 1u << j;
          break;
        case EW_GELU: y = gelu_erf_f(x); break;
        case EW_GELU_TANH: y = gelu_tanh_f<DT != DT_F32>(x); break;
        case EW_GELU_SIGMOID: y = gelu_sigmoid_f(x); break;
        case EW_RESIDUAL: y = x + opv; break;
        case EW_SCALE: y = x * P.scale; break;
        default: y = gelu_tanh_f<DT != DT_F32>(x) * opv; break;
      }
      const long long id = m * P.ldd + n;
      if (ew_in(id, P.dst_elems, P.err, code)) ew_st<DT>(P.dst, id, y);
    }
    if (P.op == EW_RELU && P.aux != nullptr) {
      const long long ia = m * P.ld_aux + w;
      if (ew_in(ia, P.aux_elems, P.err, code)) P.aux[ia] = mask;
    }
  }
}

}  // namespace fl
