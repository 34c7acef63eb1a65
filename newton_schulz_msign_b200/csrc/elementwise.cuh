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
//   ingest_kernel          cast + orient (+ scale) into the operand copy and
//                          the blocked fp32 master; optionally the fused
//                          norm (s from the unscaled copy) and the Muon
//                          momentum update (see "ingest" below).
//   apply_update_kernel    W <- W - lr * scale * O^(T) with the oriented O.
//   momentum_kernel,       the Muon momentum and update for a matrix whose
//   update_rows_kernel     msign runs as Gram NS (O stored like W).
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

// grid (kNormParts, batch); `in` holds batch matrices of `per` elements,
// matrix b starting at element b * bs.
__global__ void __launch_bounds__(kNormThreads) sumsq_partial_kernel(const void* in, int in_dt, long long per,
                                                                     long long bs, int cast_dt, float* partials) {
  __shared__ float red[32];
  const int b = blockIdx.y;
  const char* base = reinterpret_cast<const char*>(in) + static_cast<long long>(b) * bs * dtype_size(in_dt);
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

// ---------------------------------------------------------------- ingest
//
// One kernel moves a batch of input matrices into the iteration's buffers:
// cast, orient (the n x m output is in^T when `transpose`), optionally scale,
// and store the operand copy (row-major, op_dt; DT_TF32_HI writes both tf32
// planes) and the fp32 master (blocked layout of blk_off).  Work unit: a 32 x
// 64 output tile staged in shared memory.  The input is read as whole row
// segments (128 bytes per warp for 16-bit types), the operand copy is written
// as row segments, and each 32 x 32 block of the master -- one contiguous 4 KB
// span in the blocked layout -- as 256 consecutive float4 stores.  Grid
// (parts, batch), grid-stride over the tiles of a matrix, block (32, 8).
//
// Modes (fields of IngestArgs):
//   pre_scale   x = cast(in) * s[b] before the stores (fp16 operands, whose
//               range needs the normalisation first, and Gram NS).
//   partials    the fused norm: x = cast(in) is stored unscaled and the block
//               sums of x^2 go to partials; the matrix's last block (ticket
//               counter, zeroed before the launch and reset by that block)
//               sums them in a fixed order into s = 1/sqrt(sum + eps) and s^2
//               ([P2] 参考实现's normalisation, applied by the first NS step
//               in its epilogues, so the operand is rounded once), so s does
//               not depend on block timing.
//   G           Muon momentum ([P3] section 1.1): `in` is the fp32 buffer M,
//               updated in place to mu M + G before the cast.

struct IngestArgs {
  void* in;
  long long in_bs;  // elements between consecutive input matrices (0: rows * cols)
  long long ld_in;  // elements between consecutive input rows (0: cols)
  int in_dt, rows, cols, transpose, cast_dt;
  const float* pre_scale;
  void* xop;
  int op_dt;
  long long ld_op, op_bs, op_plane;
  float* master;
  long long ld_m, m_bs;
  float* partials;
  int* ticket;
  float* s_out;
  float* s2_out;
  float eps;
  const void* G;
  int g_dt;
  float mu;
};

constexpr int kIngestParts = 1024;  // blocks, and partial sums, per matrix
static_assert(kIngestParts <= kNormParts, "partials share the norm's buffer");

__device__ __forceinline__ float block_sum_lin(float v, float* red, int tid, int nthreads) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  if ((tid & 31) == 0) red[tid >> 5] = v;
  __syncthreads();
  v = (tid < (nthreads >> 5)) ? red[tid] : 0.0f;
  if (tid < 32) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  }
  __syncthreads();  // red is reused
  return v;
}

// Input element (r, c) -> x (momentum, cast, scale); 0 outside the input.
__device__ __forceinline__ float ingest_value(float x, const IngestArgs& a, float s) {
  x = round_to(x, a.cast_dt);
  return a.pre_scale ? x * s : x;
}

// Up to 8 consecutive elements p[0..cnt) of type dt (16-byte accesses when
// all 8 are wanted and p is aligned); the rest read as 0.
__device__ __forceinline__ void load8(const char* p, int dt, int cnt, float* x) {
  const int es = dtype_size(dt);
  if (cnt == 8 && (reinterpret_cast<uintptr_t>(p) & 15) == 0) {
    if (es == 4) {
      const float4 u = reinterpret_cast<const float4*>(p)[0], v = reinterpret_cast<const float4*>(p)[1];
      x[0] = u.x, x[1] = u.y, x[2] = u.z, x[3] = u.w, x[4] = v.x, x[5] = v.y, x[6] = v.z, x[7] = v.w;
    } else {
      const uint4 u = *reinterpret_cast<const uint4*>(p);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint32_t lo = w[t] & 0xFFFFu, hi = w[t] >> 16;
        if (dt == DT_BF16) {
          x[2 * t] = __uint_as_float(lo << 16), x[2 * t + 1] = __uint_as_float(hi << 16);
        } else {
          x[2 * t] = __half2float(__ushort_as_half(static_cast<unsigned short>(lo)));
          x[2 * t + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(hi)));
        }
      }
    }
    return;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = e < cnt ? load_elem(p + e * es, dt) : 0.0f;
}

// Input elements (row, col .. col+7) after the momentum update, the cast and
// the scale (ingest_value); 0 outside the input's rows x cols.
__device__ __forceinline__ void ingest_load8(const IngestArgs& a, char* src, const char* gsrc, float s, int row,
                                             int col, float* x) {
  const int cnt = (row < a.rows && col < a.cols) ? (a.cols - col < 8 ? a.cols - col : 8) : 0;
  const long long e = static_cast<long long>(row) * (a.ld_in > 0 ? a.ld_in : a.cols) + col;
  load8(src + e * dtype_size(a.in_dt), a.in_dt, cnt, x);
  if (gsrc != nullptr && cnt > 0) {
    float g[8];
    load8(gsrc + e * dtype_size(a.g_dt), a.g_dt, cnt, g);
    float* mp = reinterpret_cast<float*>(src) + e;
#pragma unroll
    for (int t = 0; t < 8; ++t) x[t] = fmaf(a.mu, x[t], g[t]);
    if (cnt == 8 && (reinterpret_cast<uintptr_t>(mp) & 15) == 0) {
      reinterpret_cast<float4*>(mp)[0] = make_float4(x[0], x[1], x[2], x[3]);
      reinterpret_cast<float4*>(mp)[1] = make_float4(x[4], x[5], x[6], x[7]);
    } else {
#pragma unroll
      for (int t = 0; t < 8; ++t)
        if (t < cnt) mp[t] = x[t];
    }
  }
#pragma unroll
  for (int t = 0; t < 8; ++t) x[t] = t < cnt ? ingest_value(x[t], a, s) : 0.0f;
}

// The values this thread owns in output tile `tt` of the non-transposed
// path: row i0 + tid/8, columns j0 + 8 (tid%8) .. +7 (0 outside the matrix).
// Tile indices fit in 32 bits (fewer than 2^31 tiles of 2048 elements for
// any matrix a device holds); 32-bit division measured 10% faster here.
__device__ __forceinline__ void ingest_row_chunk(const IngestArgs& a, char* src, const char* gsrc, float s, int tc,
                                                 long long tt, int tid, float* x) {
  const int t32 = static_cast<int>(tt);
  ingest_load8(a, src, gsrc, s, (t32 / tc) * 32 + (tid >> 3), (t32 % tc) * 64 + 8 * (tid & 7), x);
}

// Operand-copy store of 8 consecutive values at (i, j); cnt of them valid.
__device__ __forceinline__ void ingest_store_op(const IngestArgs& a, int b, int i, int j, int cnt, const float* v) {
  const int es = dtype_size(a.op_dt);
  char* dst = reinterpret_cast<char*>(a.xop) +
              (static_cast<long long>(b) * a.op_bs + static_cast<long long>(i) * a.ld_op + j) * es;
  if (cnt == 8 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
    if (es == 2) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (a.op_dt == DT_BF16) {
          __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
          w[e] = *reinterpret_cast<uint32_t*>(&h);
        } else {
          __half2 h = __floats2half2_rn(v[2 * e], v[2 * e + 1]);
          w[e] = *reinterpret_cast<uint32_t*>(&h);
        }
      }
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
      float h[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) h[e] = a.op_dt == DT_TF32_HI ? to_tf32(v[e]) : v[e];
      reinterpret_cast<float4*>(dst)[0] = make_float4(h[0], h[1], h[2], h[3]);
      reinterpret_cast<float4*>(dst)[1] = make_float4(h[4], h[5], h[6], h[7]);
      if (a.op_dt == DT_TF32_HI) {
        float4* lp = reinterpret_cast<float4*>(dst + a.op_plane * 4);
        lp[0] = make_float4(to_tf32(v[0] - h[0]), to_tf32(v[1] - h[1]), to_tf32(v[2] - h[2]), to_tf32(v[3] - h[3]));
        lp[1] = make_float4(to_tf32(v[4] - h[4]), to_tf32(v[5] - h[5]), to_tf32(v[6] - h[6]), to_tf32(v[7] - h[7]));
      }
    }
    return;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    if (e >= cnt) break;
    store_elem(dst + e * es, a.op_dt, v[e]);
    if (a.op_dt == DT_TF32_HI) store_elem(dst + a.op_plane * 4 + e * es, DT_TF32_LO, v[e]);
  }
}

// The master's part of tile (i0, j0) from the staged tile: its (up to) two
// 32 x 32 blocks, each 4 KB contiguous; thread t stores column quad t/32 of
// block row t%32 (zeros outside the matrix).
__device__ __forceinline__ void ingest_store_master(const IngestArgs& a, int b, int i0, int j0, int mpad,
                                                    const float (*tile)[65], int tid) {
  const int q = tid >> 5, r = tid & 31;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int jb = j0 + 32 * h;
    if (jb >= mpad) break;
    float* d = a.master + static_cast<long long>(b) * a.m_bs + blk_off(i0, jb, a.ld_m) + 4 * tid;
    *reinterpret_cast<float4*>(d) = make_float4(tile[r][32 * h + 4 * q], tile[r][32 * h + 4 * q + 1],
                                                tile[r][32 * h + 4 * q + 2], tile[r][32 * h + 4 * q + 3]);
  }
}

__global__ void __launch_bounds__(256, 5) ingest_kernel(const IngestArgs a) {
  __shared__ float tile[32][65];
  __shared__ float red[32];
  __shared__ int last;
  const int b = blockIdx.y;
  const int tx = threadIdx.x, ty = threadIdx.y, tid = ty * 32 + tx;
  const int n = a.transpose ? a.cols : a.rows;
  const int m = a.transpose ? a.rows : a.cols;
  const long long per = static_cast<long long>(a.rows) * a.cols;
  char* src = reinterpret_cast<char*>(a.in) + static_cast<long long>(b) * (a.in_bs > 0 ? a.in_bs : per) * dtype_size(a.in_dt);
  const char* gsrc = a.G ? reinterpret_cast<const char*>(a.G) + static_cast<long long>(b) * per * dtype_size(a.g_dt)
                         : nullptr;
  const float s = a.pre_scale ? a.pre_scale[b] : 1.0f;
  const int tr = (n + 31) / 32, tc = (m + 63) / 64;
  const long long ntiles = static_cast<long long>(tr) * tc;
  const int mpad = (m + 31) / 32 * 32;
  float acc = 0.0f;
  const long long ld_in = a.ld_in > 0 ? a.ld_in : a.cols;
  uint16_t* dop = reinterpret_cast<uint16_t*>(a.xop) + static_cast<long long>(b) * a.op_bs;
  // bf16 in and out, nothing else to do: the operand copy is the input
  // itself (its cast to bf16 is exact), moved row by row in 16-byte pieces
  // with the sum of squares on the way (the general path below spends ~40
  // instructions per element on conversions it does not need here)
  const bool copy16 = a.in_dt == DT_BF16 && a.op_dt == DT_BF16 && a.cast_dt == DT_BF16 && !a.transpose &&
                      a.pre_scale == nullptr && gsrc == nullptr && a.master == nullptr && (m & 7) == 0 &&
                      (ld_in & 7) == 0 && (a.ld_op & 7) == 0 && (a.op_bs & 7) == 0 &&
                      (reinterpret_cast<uintptr_t>(src) & 15) == 0 && (reinterpret_cast<uintptr_t>(dop) & 15) == 0;
  if (copy16) {
    // (up to four pieces, from two rows, loaded before any is stored: the
    // loads are in flight together, which the compiler cannot arrange across
    // possibly aliasing stores)
    const int mc = m >> 3;
    for (int row = blockIdx.x; row < n; row += 2 * gridDim.x) {
      const bool has2 = row + static_cast<int>(gridDim.x) < n;
      const int row2 = has2 ? row + static_cast<int>(gridDim.x) : row;
      const uint4* s0 = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(src) + row * ld_in);
      const uint4* s1 = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(src) + row2 * ld_in);
      uint4* d0 = reinterpret_cast<uint4*>(dop + row * a.ld_op);
      uint4* d1 = reinterpret_cast<uint4*>(dop + row2 * a.ld_op);
      for (int c = tid; c < mc; c += 512) {
        const bool two = c + 256 < mc;
        uint4 u[4];
        const bool ok[4] = {true, two, has2, has2 && two};
        u[0] = s0[c];
        if (ok[1]) u[1] = s0[c + 256];
        if (ok[2]) u[2] = s1[c];
        if (ok[3]) u[3] = s1[c + 256];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (!ok[q]) continue;
          (q < 2 ? d0 : d1)[c + 256 * (q & 1)] = u[q];
          const uint32_t w[4] = {u[q].x, u[q].y, u[q].z, u[q].w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float lo = __uint_as_float(w[t] << 16), hi = __uint_as_float(w[t] & 0xFFFF0000u);
            acc = fmaf(lo, lo, acc);
            acc = fmaf(hi, hi, acc);
          }
        }
      }
    }
  } else if (a.in_dt == DT_FP32 && a.op_dt == DT_BF16 && a.cast_dt == DT_BF16 && !a.transpose &&
             a.pre_scale == nullptr && a.master == nullptr && (m & 7) == 0 && (ld_in & 7) == 0 &&
             (a.ld_op & 7) == 0 && (a.op_bs & 7) == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0 &&
             (reinterpret_cast<uintptr_t>(dop) & 15) == 0 &&
             (gsrc == nullptr || (reinterpret_cast<uintptr_t>(gsrc) & 15) == 0)) {
    // fp32 in (Muon's momentum M, optionally updated by M <- mu M + G in
    // place), bf16 operands: the same row-wise walk, eight elements per step
    const int mc = m >> 3;
    for (int row = blockIdx.x; row < n; row += gridDim.x) {
      float* srow = reinterpret_cast<float*>(src) + row * ld_in;
      const char* grow = gsrc != nullptr ? gsrc + row * ld_in * dtype_size(a.g_dt) : nullptr;
      uint4* drow = reinterpret_cast<uint4*>(dop + row * a.ld_op);
      for (int c = tid; c < mc; c += 256) {
        const float4 u = reinterpret_cast<const float4*>(srow)[2 * c], v = reinterpret_cast<const float4*>(srow)[2 * c + 1];
        float x[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
        if (grow != nullptr) {
          float g[8];
          load8(grow + static_cast<long long>(8 * c) * dtype_size(a.g_dt), a.g_dt, 8, g);
#pragma unroll
          for (int t = 0; t < 8; ++t) x[t] = fmaf(a.mu, x[t], g[t]);
          reinterpret_cast<float4*>(srow)[2 * c] = make_float4(x[0], x[1], x[2], x[3]);
          reinterpret_cast<float4*>(srow)[2 * c + 1] = make_float4(x[4], x[5], x[6], x[7]);
        }
        uint32_t w[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * t], x[2 * t + 1]);
          w[t] = *reinterpret_cast<uint32_t*>(&h);
          // the norm of the rounded values, as the general path forms it
          const float lo = __uint_as_float(w[t] << 16), hi = __uint_as_float(w[t] & 0xFFFF0000u);
          acc = fmaf(lo, lo, acc);
          acc = fmaf(hi, hi, acc);
        }
        drow[c] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  } else if (!a.transpose) {
    // row chunks in registers, the next tile's loads issued before this
    // tile's stores
    float nxt[8];
    if (blockIdx.x < ntiles) ingest_row_chunk(a, src, gsrc, s, tc, blockIdx.x, tid, nxt);
    for (long long tt = blockIdx.x; tt < ntiles; tt += gridDim.x) {
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = nxt[e];
      if (tt + gridDim.x < ntiles) ingest_row_chunk(a, src, gsrc, s, tc, tt + gridDim.x, tid, nxt);
      const int i0 = (static_cast<int>(tt) / tc) * 32, j0 = (static_cast<int>(tt) % tc) * 64;
      const int r = tid >> 3, c0 = 8 * (tid & 7);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc = fmaf(v[e], v[e], acc);
      if (i0 + r < n && j0 + c0 < m) ingest_store_op(a, b, i0 + r, j0 + c0, m - j0 - c0 < 8 ? m - j0 - c0 : 8, v);
      if (a.master != nullptr) {
#pragma unroll
        for (int e = 0; e < 8; ++e) tile[r][c0 + e] = v[e];
        __syncthreads();
        if (i0 < n) ingest_store_master(a, b, i0, j0, mpad, tile, tid);
        __syncthreads();
      }
    }
  } else if (a.op_dt == DT_BF16 && a.cast_dt == DT_BF16 && a.pre_scale == nullptr && a.master == nullptr &&
             (a.in_dt == DT_BF16 || a.in_dt == DT_FP32) && (n & 7) == 0 && (ld_in & 7) == 0 &&
             (a.ld_op & 7) == 0 && (a.op_bs & 7) == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0 &&
             (reinterpret_cast<uintptr_t>(dop) & 15) == 0) {
    // transposing, bf16 operands, nothing else (tall inputs, Muon's tall
    // momenta): the tiles of the general path below without its dtype
    // dispatch per element; input rows of a multiple of 8 elements
    for (long long tt = blockIdx.x; tt < ntiles; tt += gridDim.x) {
      const int i0 = (static_cast<int>(tt) / tc) * 32, j0 = (static_cast<int>(tt) % tc) * 64;
      {
        const int jr = j0 + (tid >> 2), ic = i0 + 8 * (tid & 3);  // input row and first column
        float x[8];
        if (jr < a.rows && ic < a.cols) {
          const long long e = static_cast<long long>(jr) * ld_in + ic;
          if (a.in_dt == DT_BF16) {
            const uint4 u = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(src) + e);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int t = 0; t < 4; ++t)
              x[2 * t] = __uint_as_float(w[t] << 16), x[2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u);
          } else {
            float* mp = reinterpret_cast<float*>(src) + e;
            const float4 u = reinterpret_cast<const float4*>(mp)[0], v = reinterpret_cast<const float4*>(mp)[1];
            x[0] = u.x, x[1] = u.y, x[2] = u.z, x[3] = u.w, x[4] = v.x, x[5] = v.y, x[6] = v.z, x[7] = v.w;
            if (gsrc != nullptr) {
              float g[8];
              load8(gsrc + e * dtype_size(a.g_dt), a.g_dt, 8, g);
#pragma unroll
              for (int t = 0; t < 8; ++t) x[t] = fmaf(a.mu, x[t], g[t]);
              reinterpret_cast<float4*>(mp)[0] = make_float4(x[0], x[1], x[2], x[3]);
              reinterpret_cast<float4*>(mp)[1] = make_float4(x[4], x[5], x[6], x[7]);
            }
#pragma unroll
            for (int t = 0; t < 8; ++t) x[t] = __bfloat162float(__float2bfloat16_rn(x[t]));
          }
        } else {
#pragma unroll
          for (int t = 0; t < 8; ++t) x[t] = 0.0f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          acc = fmaf(x[e], x[e], acc);
          tile[8 * (tid & 3) + e][tid >> 2] = x[e];
        }
      }
      __syncthreads();
      const int r = tid >> 3, c0 = 8 * (tid & 7);
      if (i0 + r < n && j0 + c0 < m) {
        uint32_t w[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          __nv_bfloat162 h = __floats2bfloat162_rn(tile[r][c0 + 2 * t], tile[r][c0 + 2 * t + 1]);
          w[t] = *reinterpret_cast<uint32_t*>(&h);
        }
        uint16_t* d = dop + static_cast<long long>(i0 + r) * a.ld_op + j0 + c0;
        const int cnt = m - j0 - c0 < 8 ? m - j0 - c0 : 8;
        if (cnt == 8) {
          *reinterpret_cast<uint4*>(d) = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (e < cnt) d[e] = static_cast<uint16_t>(w[e >> 1] >> (16 * (e & 1)));
        }
      }
      __syncthreads();  // the tile is rewritten by the next iteration
    }
  } else {
    for (long long tt = blockIdx.x; tt < ntiles; tt += gridDim.x) {
      const int i0 = (static_cast<int>(tt) / tc) * 32, j0 = (static_cast<int>(tt) % tc) * 64;
      // output (i, j) = in (j, i): this thread loads input row j0 + tid/4,
      // columns i0 + 8 (tid%4) .. +7 with 16-byte accesses and stores them
      // transposed into the tile (rows padded to 65 words: the 32 lanes hit
      // 32 different banks)
      {
        float x[8];
        ingest_load8(a, src, gsrc, s, j0 + (tid >> 2), i0 + 8 * (tid & 3), x);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          acc = fmaf(x[e], x[e], acc);
          tile[8 * (tid & 3) + e][tid >> 2] = x[e];
        }
      }
      __syncthreads();
      const int r = tid >> 3, c0 = 8 * (tid & 7);
      if (i0 + r < n && j0 + c0 < m) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = tile[r][c0 + e];
        ingest_store_op(a, b, i0 + r, j0 + c0, m - j0 - c0 < 8 ? m - j0 - c0 : 8, v);
      }
      if (a.master != nullptr && i0 < n) ingest_store_master(a, b, i0, j0, mpad, tile, tid);
      __syncthreads();  // the tile is rewritten by the next iteration
    }
  }
  if (a.partials == nullptr) return;
  acc = block_sum_lin(acc, red, tid, 256);
  if (tid == 0) {
    a.partials[static_cast<long long>(b) * gridDim.x + blockIdx.x] = acc;
    __threadfence();
    last = atomicAdd(a.ticket + b, 1) == static_cast<int>(gridDim.x) - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  float v = 0.0f;
  for (int i = tid; i < static_cast<int>(gridDim.x); i += 256)
    v += __ldcg(a.partials + static_cast<long long>(b) * gridDim.x + i);
  v = block_sum_lin(v, red, tid, 256);
  if (tid == 0) {
    const float sc = 1.0f / sqrtf(v + a.eps);
    a.s_out[b] = sc;
    a.s2_out[b] = sc * sc;
    a.ticket[b] = 0;
  }
}

// ---------------------------------------------------------------- sharper initial normalisation
//
// [P2] section 改进初值 at step 0: with A = X0 X0^T and A2 = A^2 from the
// first products, n = (||A2||_F^2 + eps)^(1/8), and the step continues with
// X0 / n, A / n^2 and A2 / n^4.  Here A2 arrives as its symmetric upper
// tiles in `B` (op dtype, zero diagonal) and its diagonal in `d` (fp32), and
// ||A2||_F^2 as per-warp partials of every stored upper tile.  One block per
// (upper tile, matrix) turns them into the step's B = (b / n^2) A + (c / n^4)
// A2 in place (diagonal to d, as the BX product expects) after summing the
// matrix's partials in a fixed order; the first block of each matrix writes
// scale_out[b] = scale_in[b] / n (1 / n without scale_in), the factor BX
// applies to both its terms.  grid (nb * nb, batch, 8): z picks 32 rows of
// the tile; 256 threads.
__global__ void __launch_bounds__(256) improved_init_kernel(const void* A, void* B, int op_dt, float* d, long long ld,
                                                            long long bs, int n, int nb, const float* partials,
                                                            long long parts_bs, int slots, float bcoef, float ccoef,
                                                            float eps, const float* scale_in, float* scale_out) {
  __shared__ float red[32];
  const int b = blockIdx.y;
  const int tm = blockIdx.x / nb, tn = blockIdx.x % nb;
  if (tm > tn) return;
  const int tid = threadIdx.x;
  // ||A2||_F^2: the partials of the upper tiles, in a fixed order
  float v = 0.0f;
  const float* pp = partials + static_cast<long long>(b) * parts_bs;
  for (int i = tid; i < nb * nb * slots; i += 256) {
    const int t = i / slots;
    if (t / nb <= t % nb) v += pp[i];
  }
  v = block_sum_lin(v, red, tid, 256);
  __shared__ float s_n;
  if (tid == 0) s_n = sqrtf(sqrtf(sqrtf(v + eps)));  // (sum + eps)^(1/8)
  __syncthreads();
  const float nn = s_n;
  const float kb = bcoef / (nn * nn), kc = ccoef / (nn * nn * nn * nn);
  if (blockIdx.x == 0 && blockIdx.z == 0 && tid == 0) scale_out[b] = (scale_in ? scale_in[b] : 1.0f) / nn;
  const char* ab = reinterpret_cast<const char*>(A) + static_cast<long long>(b) * bs * dtype_size(op_dt);
  char* bb = reinterpret_cast<char*>(B) + static_cast<long long>(b) * bs * dtype_size(op_dt);
  float* db = d + static_cast<long long>(b) * n;
  const int r0 = tm * 256 + 32 * blockIdx.z, c0 = tn * 256;
  for (int e = tid; e < 32 * 256; e += 256) {
    const int i = r0 + e / 256, j = c0 + e % 256;
    if (i >= n || j >= n) continue;
    const long long off = static_cast<long long>(i) * ld + j;
    const float a = load_elem(ab + off * dtype_size(op_dt), op_dt);
    if (i == j) {
      db[i] = kb * a + kc * db[i];
    } else {
      char* q = bb + off * dtype_size(op_dt);
      store_elem(q, op_dt, kb * a + kc * load_elem(q, op_dt));
    }
  }
}

// ---------------------------------------------------------------- Mousse preconditioner roots
//
// Start of the coupled Newton iteration for (A + eps I)^(-1/4), the inverse
// fourth roots of the Mousse post's Kronecker factors: with
// s = 1 / (||A||_F + eps) (s_in[b]) the scaled matrix M0 = s (A + eps I) has
// its eigenvalues in (0, 1], and the first iterate is X1 = X0 (5 I - M0) / 4
// with X0 = s^(1/4) I.  Only the upper triangle of A is read (the lower one
// is taken as its mirror), so M0 is exactly symmetric.  Both matrices are
// stored as tf32 (hi, lo) plane pairs for the fp32-accurate products: matrix
// b at element 2 b plane, the lo plane `plane` elements after the hi plane,
// rows ld apart.  Grid (blocks, batch), grid-stride over the n x n elements.
__global__ void __launch_bounds__(256) inv_root_start_kernel(const float* A, int n, long long a_bs, const float* s_in,
                                                             float eps, float* M, float* X, long long ld,
                                                             long long plane) {
  const int b = blockIdx.y;
  const float s = s_in[b];
  const float q = sqrtf(sqrtf(s));
  const float* a = A + static_cast<long long>(b) * a_bs;
  float* mh = M + 2 * plane * b;
  float* xh = X + 2 * plane * b;
  const long long total = static_cast<long long>(n) * n;
  for (long long e = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * 256) {
    const int i = static_cast<int>(e / n), j = static_cast<int>(e % n);
    const float aij = i <= j ? a[e] : a[static_cast<long long>(j) * n + i];
    const float m0 = s * (aij + (i == j ? eps : 0.0f));
    const float x1 = q * ((i == j ? 5.0f : 0.0f) - m0) * 0.25f;
    const long long o = static_cast<long long>(i) * ld + j;
    const float mhi = to_tf32(m0), xhi = to_tf32(x1);
    mh[o] = mhi;
    mh[o + plane] = to_tf32(m0 - mhi);
    xh[o] = xhi;
    xh[o + plane] = to_tf32(x1 - xhi);
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

// Stores cnt <= 8 consecutive values in dt (16-byte stores when whole and
// aligned), rounding to nearest even like store_elem.
__device__ __forceinline__ void store8(char* p, int dt, int cnt, const float* v) {
  if (cnt == 8 && (reinterpret_cast<uintptr_t>(p) & 15) == 0) {
    if (dt == DT_FP32) {
      reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
      reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
      uint32_t w[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint32_t lo = dt == DT_BF16 ? __bfloat16_as_ushort(__float2bfloat16_rn(v[2 * t]))
                                          : __half_as_ushort(__float2half_rn(v[2 * t]));
        const uint32_t hi = dt == DT_BF16 ? __bfloat16_as_ushort(__float2bfloat16_rn(v[2 * t + 1]))
                                          : __half_as_ushort(__float2half_rn(v[2 * t + 1]));
        w[t] = lo | (hi << 16);
      }
      *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    return;
  }
  const int es = dtype_size(dt);
  for (int e = 0; e < cnt; ++e) store_elem(p + e * es, dt, v[e]);
}

// M <- mu M + G, elementwise over n fp32 values (G in g_dt): the Muon
// momentum of a matrix whose msign runs as Gram NS.  The same fused
// multiply-add as the standard route's ingest; 8 values per thread step.
__global__ void __launch_bounds__(256) momentum_kernel(float* M, const void* G, int g_dt, float mu, long long n) {
  const char* g = static_cast<const char*>(G);
  const int es = dtype_size(g_dt);
  const long long chunks = (n + 7) / 8;
  for (long long c = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; c < chunks;
       c += static_cast<long long>(gridDim.x) * 256) {
    const long long e = 8 * c;
    const int cnt = static_cast<int>(n - e < 8 ? n - e : 8);
    float m[8], gv[8];
    load8(reinterpret_cast<const char*>(M + e), DT_FP32, cnt, m);
    load8(g + e * es, g_dt, cnt, gv);
#pragma unroll
    for (int t = 0; t < 8; ++t) m[t] = fmaf(mu, m[t], gv[t]);
    store8(reinterpret_cast<char*>(M + e), DT_FP32, cnt, m);
  }
}

// W <- W - coef * O, elementwise over n values, O (o_dt) stored like W
// (w_dt); the same arithmetic as apply_update_kernel; 8 values per thread
// step.
__global__ void __launch_bounds__(256) update_rows_kernel(void* W, int w_dt, const void* O, int o_dt, float coef,
                                                          long long n) {
  char* w = static_cast<char*>(W);
  const char* o = static_cast<const char*>(O);
  const int ew = dtype_size(w_dt), eo = dtype_size(o_dt);
  const long long chunks = (n + 7) / 8;
  for (long long c = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; c < chunks;
       c += static_cast<long long>(gridDim.x) * 256) {
    const long long e = 8 * c;
    const int cnt = static_cast<int>(n - e < 8 ? n - e : 8);
    float wv[8], ov[8];
    load8(w + e * ew, w_dt, cnt, wv);
    load8(o + e * eo, o_dt, cnt, ov);
#pragma unroll
    for (int t = 0; t < 8; ++t) wv[t] = wv[t] - coef * ov[t];
    store8(w + e * ew, w_dt, cnt, wv);
  }
}

}  // namespace msb
