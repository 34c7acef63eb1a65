// elementwise.cuh - the HBM-bound steps around the tensor-core loop.
//
//   sumsq_partial_kernel   per-matrix sum of squares of the (compute-dtype
//                          cast) input: grid-stride, 16-byte loads, warp
//                          shuffle + block reduction into one partial per
//                          block (no atomics: the result is deterministic);
//                          the grid grows with the matrix to keep HBM busy.
//   norm_finalize_kernel   sums the partials in a fixed order and writes the
//                          normalisation factor of [P2] section 参考实现
//                          (1/sqrt(sum + eps)) or of [P3] Algorithm 2 step 1
//                          (1/(sqrt(sum) + eps)).
//   ingest_kernel          cast + orient + scale: X0 = cast(cast(M) * s),
//                          transposed through a 32x32 shared-memory tile
//                          when rows > cols, plus the fp32 copy of X0;
//   ingest_rows_kernel     the same without transposition, 16-byte accesses.
//                          With op_dt DT_TF32_HI both write the two tf32
//                          planes (hi, lo) of the fp32-accurate operand.
//   momentum_kernel        M <- mu M + G in fp32 (Muon, [P3] section 1.1).
//   apply_update_kernel    W <- W - lr * scale * O^(T) with the oriented O.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "gemm_sm100.cuh"

namespace msb {

constexpr int kNormParts = 2048;  // maximum partial sums per matrix
constexpr int kNormThreads = 256;
constexpr int kNormElemsPerBlock = kNormThreads * 16;  // 16 elements per thread per pass

// Blocks per matrix for the sum of squares: enough to keep HBM busy, at most kNormParts.
__host__ __device__ inline int norm_parts(long long per) {
  long long b = (per + kNormElemsPerBlock - 1) / kNormElemsPerBlock;
  return static_cast<int>(b < 1 ? 1 : (b > kNormParts ? kNormParts : b));
}

// Rounds v to the compute dtype (bf16 / fp16) and back; DT_FP32 keeps it.
__device__ __forceinline__ float round_to(float v, int dt) {
  if (dt == DT_BF16) return __bfloat162float(__float2bfloat16_rn(v));
  if (dt == DT_FP16) return __half2float(__float2half_rn(v));
  return v;
}

__device__ __forceinline__ float block_reduce_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  const int nw = blockDim.x >> 5;
  v = (threadIdx.x < nw) ? red[threadIdx.x] : 0.0f;
  if (warp == 0) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  }
  return v;
}

// grid (kNormParts, batch); `in` holds batch matrices of `per` elements.
__global__ void __launch_bounds__(kNormThreads) sumsq_partial_kernel(const void* in, int in_dt, long long per,
                                                                     int cast_dt, float* partials) {
  __shared__ float red[32];
  const int b = blockIdx.y;
  const char* base = reinterpret_cast<const char*>(in) + static_cast<long long>(b) * per * dtype_size(in_dt);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  float acc = 0.0f;
  const bool vec = (reinterpret_cast<uintptr_t>(base) & 15) == 0;
  if (vec && in_dt == DT_FP32) {
    const long long nv = per / 4;
    for (long long i = blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride) {
      float4 f = reinterpret_cast<const float4*>(base)[i];
      float a = round_to(f.x, cast_dt), c = round_to(f.y, cast_dt), d = round_to(f.z, cast_dt),
            e = round_to(f.w, cast_dt);
      acc += a * a + c * c + d * d + e * e;
    }
    for (long long i = nv * 4 + blockIdx.x * blockDim.x + threadIdx.x; i < per; i += stride) {
      float a = round_to(reinterpret_cast<const float*>(base)[i], cast_dt);
      acc += a * a;
    }
  } else if (vec) {
    const long long nv = per / 8;
    for (long long i = blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride) {
      uint4 u = reinterpret_cast<const uint4*>(base)[i];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 f;
        if (in_dt == DT_BF16)
          f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
        else
          f = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
        float a = round_to(f.x, cast_dt), c = round_to(f.y, cast_dt);
        acc += a * a + c * c;
      }
    }
    for (long long i = nv * 8 + blockIdx.x * blockDim.x + threadIdx.x; i < per; i += stride) {
      float a = round_to(load_elem(base + i * 2, in_dt), cast_dt);
      acc += a * a;
    }
  } else {
    const int es = dtype_size(in_dt);
    for (long long i = blockIdx.x * blockDim.x + threadIdx.x; i < per; i += stride) {
      float a = round_to(load_elem(base + i * es, in_dt), cast_dt);
      acc += a * a;
    }
  }
  acc = block_reduce_sum(acc, red);
  if (threadIdx.x == 0) partials[static_cast<long long>(b) * gridDim.x + blockIdx.x] = acc;
}

// One block of 1024 threads per matrix sums the nparts partials in a fixed
// order.  mode 0: s = 1/sqrt(sum + eps); mode 1: s = 1/(sqrt(sum) + eps).
__global__ void __launch_bounds__(1024) norm_finalize_kernel(const float* partials, int nparts, float eps,
                                                             int mode, float* scale) {
  __shared__ float red[32];
  const int b = blockIdx.x;
  float v = 0.0f;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) v += partials[static_cast<long long>(b) * nparts + i];
  v = block_reduce_sum(v, red);
  if (threadIdx.x == 0) {
    const float s = (mode == 0) ? 1.0f / sqrtf(v + eps) : 1.0f / (sqrtf(v) + eps);
    scale[b] = s;
  }
}

// Output space: n x m per matrix (n = rows, m = cols, or swapped when
// `transpose`).  Block (32, 8) handles a 32 x 32 output tile.
//   xop[i][j]    = round_op(cast(in) * s)      (operand copy, op_dt)
//   master(i, j) = cast(in) * s                 (fp32 copy, blocked layout
//                                                with padded width ld_m; nullable)
// in[b] is rows x cols row-major with leading dimension `cols`.
__global__ void __launch_bounds__(256) ingest_kernel(const void* in, int in_dt, int rows, int cols, int transpose,
                                                     const float* scale, int cast_dt, void* xop, int op_dt,
                                                     long long ld_op, long long op_bs, long long op_plane,
                                                     float* master, long long ld_m, long long m_bs) {
  __shared__ float tile[32][33];
  const int b = blockIdx.z;
  const int n = transpose ? cols : rows;
  const int m = transpose ? rows : cols;
  const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  const char* src = reinterpret_cast<const char*>(in) +
                    static_cast<long long>(b) * rows * static_cast<long long>(cols) * dtype_size(in_dt);
  const float s = scale ? scale[b] : 1.0f;
  float v[4];
  if (!transpose) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = i0 + ty + 8 * k, j = j0 + tx;
      v[k] = (i < n && j < m)
                 ? round_to(load_elem(src + (static_cast<long long>(i) * cols + j) * dtype_size(in_dt), in_dt),
                            cast_dt)
                 : 0.0f;
    }
  } else {
    // out(i, j) = in(j, i): read rows j0.. of `in` along its columns i0..
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int jr = j0 + ty + 8 * k, ic = i0 + tx;
      tile[ty + 8 * k][tx] =
          (jr < m && ic < n)
              ? round_to(load_elem(src + (static_cast<long long>(jr) * cols + ic) * dtype_size(in_dt), in_dt),
                         cast_dt)
              : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = tile[tx][ty + 8 * k];
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = i0 + ty + 8 * k, j = j0 + tx;
    if (i < n && j < m) {
      const float xs = v[k] * s;
      char* dst = reinterpret_cast<char*>(xop) +
                  (static_cast<long long>(b) * op_bs + static_cast<long long>(i) * ld_op + j) * dtype_size(op_dt);
      store_elem(dst, op_dt, xs);
      if (op_dt == DT_TF32_HI) store_elem(dst + op_plane * 4, DT_TF32_LO, xs);
      if (master) master[static_cast<long long>(b) * m_bs + blk_off(i, j, ld_m)] = xs;
    }
  }
}

// Row-wise ingest without transposition, 8 elements per thread with 16-byte
// accesses: rows x cols input (leading dimension cols) to the operand copy and
// the fp32 copy (leading dimensions ld_op, ld_m).  Requires cols % 8 == 0 and
// 16-byte aligned bases and rows on every side.
template <int IN_DT, int OP_DT>
__global__ void __launch_bounds__(256) ingest_rows_kernel(const void* in, long long rows, int cols,
                                                          const float* scale, int cast_dt, void* xop, long long ld_op,
                                                          long long op_bs, long long op_plane, float* master,
                                                          long long ld_m, long long m_bs) {
  const int b = blockIdx.y;
  const int vpr = cols / 8;  // vectors per row
  const long long nvec = rows * vpr;
  const float s = scale ? scale[b] : 1.0f;
  const char* src = reinterpret_cast<const char*>(in) + static_cast<long long>(b) * rows * cols * dtype_size(IN_DT);
  for (long long v = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; v < nvec;
       v += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long i = v / vpr;
    const int j = static_cast<int>(v - i * vpr) * 8;
    float x[8];
    if (IN_DT == DT_FP32) {
      const float4* q = reinterpret_cast<const float4*>(src + (i * cols + j) * 4);
      const float4 a = q[0], c = q[1];
      x[0] = a.x, x[1] = a.y, x[2] = a.z, x[3] = a.w, x[4] = c.x, x[5] = c.y, x[6] = c.z, x[7] = c.w;
    } else {
      const uint4 u = *reinterpret_cast<const uint4*>(src + (i * cols + j) * 2);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float2 f;
        if (IN_DT == DT_BF16)
          f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[t]));
        else
          f = __half22float2(*reinterpret_cast<const __half2*>(&w[t]));
        x[2 * t] = f.x, x[2 * t + 1] = f.y;
      }
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) x[t] = round_to(x[t], cast_dt) * s;
    if (OP_DT == DT_TF32_HI) {
      // fp32-accurate operand: tf32 hi plane and tf32 lo plane
      float* hp = reinterpret_cast<float*>(xop) + static_cast<long long>(b) * op_bs + i * ld_op + j;
      float h[8], l[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        h[t] = to_tf32(x[t]);
        l[t] = to_tf32(x[t] - h[t]);
      }
      reinterpret_cast<float4*>(hp)[0] = make_float4(h[0], h[1], h[2], h[3]);
      reinterpret_cast<float4*>(hp)[1] = make_float4(h[4], h[5], h[6], h[7]);
      reinterpret_cast<float4*>(hp + op_plane)[0] = make_float4(l[0], l[1], l[2], l[3]);
      reinterpret_cast<float4*>(hp + op_plane)[1] = make_float4(l[4], l[5], l[6], l[7]);
      if (master) {
        float* d = master + static_cast<long long>(b) * m_bs + blk_off(i, j, ld_m);
        *reinterpret_cast<float4*>(d) = make_float4(x[0], x[1], x[2], x[3]);
        *reinterpret_cast<float4*>(d + 128) = make_float4(x[4], x[5], x[6], x[7]);
      }
      continue;
    }
    uint32_t o[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      if (OP_DT == DT_BF16) {
        __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * t], x[2 * t + 1]);
        o[t] = *reinterpret_cast<uint32_t*>(&h);
      } else {
        __half2 h = __floats2half2_rn(x[2 * t], x[2 * t + 1]);
        o[t] = *reinterpret_cast<uint32_t*>(&h);
      }
    }
    *reinterpret_cast<uint4*>(reinterpret_cast<char*>(xop) + (static_cast<long long>(b) * op_bs + i * ld_op + j) * 2) =
        make_uint4(o[0], o[1], o[2], o[3]);
    if (master) {
      float* d = master + static_cast<long long>(b) * m_bs + blk_off(i, j, ld_m);
      *reinterpret_cast<float4*>(d) = make_float4(x[0], x[1], x[2], x[3]);
      *reinterpret_cast<float4*>(d + 128) = make_float4(x[4], x[5], x[6], x[7]);
    }
  }
}

// M <- mu * M + G over `count` elements (fp32 M, G in g_dt).
__global__ void __launch_bounds__(256) momentum_kernel(float* M, const void* G, int g_dt, long long count, float mu) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const bool vec = ((reinterpret_cast<uintptr_t>(M) | reinterpret_cast<uintptr_t>(G)) & 15) == 0 && g_dt == DT_FP32;
  if (vec) {
    const long long nv = count / 4;
    for (long long i = blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride) {
      float4 m = reinterpret_cast<float4*>(M)[i];
      const float4 g = reinterpret_cast<const float4*>(G)[i];
      m.x = fmaf(mu, m.x, g.x);
      m.y = fmaf(mu, m.y, g.y);
      m.z = fmaf(mu, m.z, g.z);
      m.w = fmaf(mu, m.w, g.w);
      reinterpret_cast<float4*>(M)[i] = m;
    }
    for (long long i = nv * 4 + blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride)
      M[i] = fmaf(mu, M[i], reinterpret_cast<const float*>(G)[i]);
  } else {
    const int es = dtype_size(g_dt);
    for (long long i = blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride)
      M[i] = fmaf(mu, M[i], load_elem(reinterpret_cast<const char*>(G) + i * es, g_dt));
  }
}

// W (rows x cols, w_dt) <- W - coef * O where O is stored oriented:
// n x m in the blocked fp32 layout of padded width ld_o, transposed when
// `transpose`.
__global__ void __launch_bounds__(256) apply_update_kernel(void* W, int w_dt, int rows, int cols, const float* O,
                                                           long long ld_o, int transpose, float coef) {
  __shared__ float tile[32][33];
  const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;  // W tile
  const int tx = threadIdx.x, ty = threadIdx.y;
  float o[4];
  if (!transpose) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = i0 + ty + 8 * k, j = j0 + tx;
      o[k] = (i < rows && j < cols) ? O[blk_off(i, j, ld_o)] : 0.0f;
    }
  } else {
    // W(i, j) -= O(j, i): O is cols x rows
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int orow = j0 + ty + 8 * k, ocol = i0 + tx;
      tile[ty + 8 * k][tx] = (orow < cols && ocol < rows) ? O[blk_off(orow, ocol, ld_o)] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 4; ++k) o[k] = tile[tx][ty + 8 * k];
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = i0 + ty + 8 * k, j = j0 + tx;
    if (i < rows && j < cols) {
      char* p = reinterpret_cast<char*>(W) + (static_cast<long long>(i) * cols + j) * dtype_size(w_dt);
      store_elem(p, w_dt, load_elem(p, w_dt) - coef * o[k]);
    }
  }
}

}  // namespace msb
