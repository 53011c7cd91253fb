// fl_elementwise.cuh — HBM-bound kernels of the fused linear layer:
//
//   * fl_relu_backward_kernel: dpre = grad ⊙ bit(mask), the backward use of the
//     RELU_AUX_BIAS mask (cuBLASLt epilog page: the aux ReLU mask serves the
//     backward pass).  One thread per (row, 32-column mask word): one 4-byte
//     mask load and 32 contiguous elements in 16-byte vectors.
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

// ---------------------------------------------------------------- dReLU
template <int DT>
__global__ void __launch_bounds__(256) fl_relu_backward_kernel(const void* __restrict__ grad_,
                                                               const uint32_t* __restrict__ aux,
                                                               void* __restrict__ dpre_, long long M,
                                                               long long N, long long ldg,
                                                               long long ldd, long long words,
                                                               int vec_ok) {
  using T = typename ElemT<DT>::T;
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  constexpr int ESZ = sizeof(T);
  constexpr int PER16 = 16 / ESZ;  // elements per 16-byte vector
  const T* grad = reinterpret_cast<const T*>(grad_);
  T* dpre = reinterpret_cast<T*>(dpre_);
  const int lane = threadIdx.x & 31;
  // A warp takes a block of 32 mask words (32·32 elements) of one row.  In a full
  // block lane l moves 16-byte vectors l, l+32, ... of the block, so every warp-wide
  // access is 512 contiguous bytes, and reads its mask bits from the block's 32 words
  // (one coalesced load) by shuffle.
  const long long wblocks = (words + 31) / 32;
  const long long total = M * wblocks;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long blk = warp0; blk < total; blk += nwarps) {
    const long long m = blk / wblocks;
    const long long w0 = (blk - m * wblocks) * 32;
    const T* g = grad + m * ldg + w0 * 32;
    T* d = dpre + m * ldd + w0 * 32;
    const uint32_t myword = (w0 + lane < words) ? __ldg(aux + m * words + w0 + lane) : 0u;
    if (vec_ok && w0 + 32 <= words && (w0 + 32) * 32 <= N) {
#pragma unroll
      for (int v = 0; v < 32 * 32 / PER16 / 32; ++v) {
        const int e0 = (v * 32 + lane) * PER16;  // first element of this lane's vector
        const uint32_t bits = __shfl_sync(0xffffffffu, myword, e0 >> 5);
        uint4 x = __ldg(reinterpret_cast<const uint4*>(g) + v * 32 + lane);
        uint32_t* xw = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if constexpr (ESZ == 2) {
            const int j = (e0 & 31) + e * 2;
            // grad·0 keeps the sign of grad (IEEE): clear all but the sign bit
            const uint32_t lo_keep = ((bits >> j) & 1u) ? 0x0000FFFFu : 0x00008000u;
            const uint32_t hi_keep = ((bits >> (j + 1)) & 1u) ? 0xFFFF0000u : 0x80000000u;
            xw[e] &= (lo_keep | hi_keep);
          } else {
            const int j = (e0 & 31) + e;
            xw[e] &= ((bits >> j) & 1u) ? 0xFFFFFFFFu : 0x80000000u;
          }
        }
        reinterpret_cast<uint4*>(d)[v * 32 + lane] = x;
      }
    } else {
      // ragged block: lane l finishes word w0 + l element by element
      const long long w = w0 + lane;
      if (w < words) {
        const long long n0 = w * 32;
        for (int j = 0; j < 32 && n0 + j < N; ++j) {
          T x = g[lane * 32 + j];
          if (!((myword >> j) & 1u)) {
            if constexpr (ESZ == 2) {
              unsigned short b = *reinterpret_cast<unsigned short*>(&x);
              b &= 0x8000u;
              x = *reinterpret_cast<T*>(&b);
            } else {
              uint32_t b = __float_as_uint(x) & 0x80000000u;
              x = __uint_as_float(b);
            }
          }
          d[lane * 32 + j] = x;
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
  EW_GEGLU_MUL = 7 // y[m,n] = gelu_tanh(x[m,n]) * u[m,n]  (u = operand)
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

// Storage dtype DT for src/dst (the eager tensors); operands use their own dtype.
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
