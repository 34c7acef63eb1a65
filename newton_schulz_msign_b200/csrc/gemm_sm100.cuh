// gemm_sm100.cuh - persistent, warp-specialised tcgen05 GEMM engine with
// the fused epilogues of the Newton-Schulz family.
//
// One launch computes D = epilogue(A_op * B_op^T) for every tile of up to
// kMaxClasses "classes"; a class is a batch of same-shape problems whose
// operands are 3-D TMA tensors (k, row, batch).  The tile list is the
// concatenation of the classes' tiles (the host orders classes by K, longest
// first, so short tiles fill the tail of the last wave).
//
// Roles inside a 192-thread CTA (one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: fills a kStages-deep ring of 128-byte-swizzled
//               shared-memory stages (A 128x64, B 256x64 elements).
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators)
//               and issues tcgen05.mma (M=128, N=256, K=16) from one thread;
//               tcgen05.commit releases a stage / publishes an accumulator.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4)..+31 = tile rows), fused arithmetic
//               v = alpha*acc + beta*C, then up to kMaxOuts stores, each
//               direct or transposed (through a padded shared-memory
//               transpose) and each with its own gamma*I diagonal term.
//
// Symmetric classes ([P1] flash-muon matmul_transpose; [P3] section 4,
// triangular scheduler) enumerate only tiles that touch the upper triangle
// (tile (tm, tn) with tn >= tm/2 for 128x256 tiles).  In them, 32x32 blocks
// strictly below the diagonal are skipped, blocks above it are stored
// directly and transposed into the mirrored position, and diagonal blocks
// store their upper part directly and their strict upper part transposed.
// Both copies come from the same fp32 value with the same rounding, so the
// stored matrix is bit-exactly symmetric.
//
// The B operand is read K-major (rows of B_op are the output columns) or
// MN-major (B_op^T stored row-major as K x N, e.g. X in B*X), the latter via
// the UMMA descriptor's MN-major mode, so X is never transposed in memory.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx_sm100.cuh"

namespace msb {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;  // 64 16-bit elements = one 128-byte swizzle row
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kATileBytes = kBM * kBK * 2;  // 16 KB
constexpr int kBTileBytes = kBN * kBK * 2;  // 32 KB
constexpr int kStageBytes = kATileBytes + kBTileBytes;
constexpr int kEpiStride = 33;  // padded row of the 32x32 transpose buffer
constexpr int kEpiWarpFloats = 32 * kEpiStride;
constexpr int kTmemCols = 512;
constexpr int kMaxClasses = 8;
constexpr int kNumBarriers = 2 * kStages + 2 + 2 + 1;
constexpr int kSmemBytes = 1024 /* alignment slack */ + kStages * kStageBytes + 4 * kEpiWarpFloats * 4 +
                           kNumBarriers * 8 + 16;

enum : int { DT_BF16 = 0, DT_FP16 = 1, DT_FP32 = 2 };

__host__ __device__ inline int dtype_size(int dt) { return dt == DT_FP32 ? 4 : 2; }

// One epilogue output.  Direct: D[row][col] = w; transposed: D[col][row] = w,
// where w = v + gamma * [row == col] and v = alpha*acc + beta*C.
struct EpiOut {
  void* ptr;
  long long ld, bs;  // leading dimension and batch stride, in elements
  int dtype;
  int transposed;
  float gamma;
  int pad;
};

constexpr int kMaxOuts = 4;

struct alignas(64) GemmClass {
  CUtensorMap tmA;  // (k, row, batch), K-major, box 64 x 128
  CUtensorMap tmB;  // K-major: (k, col, batch) box 64 x 256; MN-major: (col, k, batch) box 64 x 64
  int M, N, K, batch;
  int tiles_m, tiles_n, tiles_per_batch, tile_begin;
  int symmetric, b_mn_major, num_out, pad0;
  float alpha, beta;
  const float* alpha_scale;  // optional per-batch factor on alpha
  const float* beta_scale;   // optional per-batch factor on beta
  const void* C;             // optional epilogue input, C[row][col]
  long long ldc, c_bs;
  int c_dtype, pad1;
  EpiOut out[kMaxOuts];
};

struct GemmParams {
  GemmClass cls[kMaxClasses];
  int num_classes;
  int total_tiles;
  uint32_t idesc;  // instruction descriptor without the B-major bit
  int* err;        // device error word (bit 0: a bounded wait ran out)
  unsigned long long timeout_ns;
};

struct TileCoord {
  int c, b, tm, tn;
};

__device__ __forceinline__ TileCoord decode_tile(const GemmParams& p, int t) {
  int c = 0;
  while (c + 1 < p.num_classes && t >= p.cls[c + 1].tile_begin) ++c;
  const GemmClass& k = p.cls[c];
  int l = t - k.tile_begin;
  int b = l / k.tiles_per_batch;
  int r = l - b * k.tiles_per_batch;
  int tm, tn;
  if (!k.symmetric) {
    tm = r / k.tiles_n;
    tn = r - tm * k.tiles_n;
  } else {
    tm = 0;
    while (true) {
      int cnt = k.tiles_n - (tm >> 1);
      if (r < cnt) break;
      r -= cnt;
      ++tm;
    }
    tn = (tm >> 1) + r;
  }
  return {c, b, tm, tn};
}

// ---------------------------------------------------------------- row I/O

__device__ __forceinline__ float load_elem(const char* p, int dt) {
  if (dt == DT_FP32) return *reinterpret_cast<const float*>(p);
  if (dt == DT_BF16) return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
  return __half2float(*reinterpret_cast<const __half*>(p));
}

__device__ __forceinline__ void store_elem(char* p, int dt, float v) {
  if (dt == DT_FP32)
    *reinterpret_cast<float*>(p) = v;
  else if (dt == DT_BF16)
    *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(v);
  else
    *reinterpret_cast<__half*>(p) = __float2half_rn(v);
}

// Loads 32 consecutive elements of one row; lanes outside `mask` read 0.
__device__ __forceinline__ void load_row32(const char* rowp, int dt, uint32_t mask, float (&v)[32]) {
  const int es = dtype_size(dt);
  if (mask == 0xFFFFFFFFu && (reinterpret_cast<uintptr_t>(rowp) & 15) == 0) {
    if (dt == DT_FP32) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float4 f = reinterpret_cast<const float4*>(rowp)[i];
        v[4 * i + 0] = f.x;
        v[4 * i + 1] = f.y;
        v[4 * i + 2] = f.z;
        v[4 * i + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 u = reinterpret_cast<const uint4*>(rowp)[i];
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (dt == DT_BF16) {
            __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&w[j]);
            float2 f = __bfloat1622float2(h);
            v[8 * i + 2 * j] = f.x;
            v[8 * i + 2 * j + 1] = f.y;
          } else {
            __half2 h = *reinterpret_cast<__half2*>(&w[j]);
            float2 f = __half22float2(h);
            v[8 * i + 2 * j] = f.x;
            v[8 * i + 2 * j + 1] = f.y;
          }
        }
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = ((mask >> i) & 1u) ? load_elem(rowp + i * es, dt) : 0.0f;
  }
}

// Stores the elements of `v` selected by `mask` to 32 consecutive row slots.
__device__ __forceinline__ void store_row32(char* rowp, int dt, uint32_t mask, const float (&v)[32]) {
  const int es = dtype_size(dt);
  if (mask == 0xFFFFFFFFu && (reinterpret_cast<uintptr_t>(rowp) & 15) == 0) {
    if (dt == DT_FP32) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        reinterpret_cast<float4*>(rowp)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (dt == DT_BF16) {
            __nv_bfloat162 h = __floats2bfloat162_rn(v[8 * i + 2 * j], v[8 * i + 2 * j + 1]);
            w[j] = *reinterpret_cast<uint32_t*>(&h);
          } else {
            __half2 h = __floats2half2_rn(v[8 * i + 2 * j], v[8 * i + 2 * j + 1]);
            w[j] = *reinterpret_cast<uint32_t*>(&h);
          }
        }
        reinterpret_cast<uint4*>(rowp)[i] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if ((mask >> i) & 1u) store_elem(rowp + i * es, dt, v[i]);
  }
}

__device__ __forceinline__ char* row_ptr(void* base, int dt, long long ld, long long bs, int b, long long r,
                                         long long c) {
  return reinterpret_cast<char*>(base) + (static_cast<long long>(b) * bs + r * ld + c) * dtype_size(dt);
}

// ---------------------------------------------------------------- epilogue

// One 32x32 block: this lane owns output row `row0 + lane`, columns
// col0..col0+31, whose fp32 accumulators are in `acc`.
__device__ __forceinline__ void epilogue_block(const GemmClass& k, int b, int row0, int col0, float (&acc)[32],
                                               float* stage, int lane) {
  const int r = row0 + lane;
  const bool diag = k.symmetric && (col0 == row0);
  const uint32_t colmask = (k.N - col0 >= 32) ? 0xFFFFFFFFu : ((1u << (k.N - col0)) - 1u);
  const uint32_t rowmask = (k.M - row0 >= 32) ? 0xFFFFFFFFu : ((1u << (k.M - row0)) - 1u);

  float alpha = k.alpha;
  if (k.alpha_scale != nullptr) alpha *= k.alpha_scale[b];
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] *= alpha;

  if (k.C != nullptr) {
    float beta = k.beta;
    if (k.beta_scale != nullptr) beta *= k.beta_scale[b];
    float cv[32];
    const uint32_t m = (r < k.M) ? colmask : 0u;
    load_row32(row_ptr(const_cast<void*>(k.C), k.c_dtype, k.ldc, k.c_bs, b, r, col0), k.c_dtype, m, cv);
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = fmaf(beta, cv[i], acc[i]);
  }

#pragma unroll 1
  for (int o = 0; o < k.num_out; ++o) {
    const EpiOut& e = k.out[o];
    float w[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i] = (col0 + i == r) ? acc[i] + e.gamma : acc[i];
    if (!e.transposed) {
      if (r < k.M) {
        uint32_t m = colmask;
        if (diag) m &= (0xFFFFFFFFu << lane);  // keep columns c >= r
        store_row32(row_ptr(e.ptr, e.dtype, e.ld, e.bs, b, r, col0), e.dtype, m, w);
      }
    } else {
      // stage[i][lane] = w(row0 + lane, col0 + i); read back transposed so
      // that lane l owns row col0 + l of D, columns row0..row0+31.
#pragma unroll
      for (int i = 0; i < 32; ++i) stage[i * kEpiStride + lane] = w[i];
      __syncwarp();
      float t[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) t[j] = stage[lane * kEpiStride + j];
      __syncwarp();
      const int tr = col0 + lane;
      if (tr < k.N) {
        uint32_t m = rowmask;
        if (diag) m &= (lane == 0) ? 0u : (0xFFFFFFFFu >> (32 - lane));  // keep rows r < c (strict)
        store_row32(row_ptr(e.ptr, e.dtype, e.ld, e.bs, b, tr, row0), e.dtype, m, t);
      }
    }
  }
}

// ---------------------------------------------------------------- kernel

__global__ void __launch_bounds__(kThreads, 1) gemm_sm100_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kATileBytes;
  float* sEpi = reinterpret_cast<float*>(sB + kStages * kBTileBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + 4 * kEpiWarpFloats);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* tfull = bars + 2 * kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + kNumBarriers);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t limit = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4 * 32);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    for (int c = 0; c < p.num_classes; ++c) {
      tma_prefetch_desc(&p.cls[c].tmA);
      tma_prefetch_desc(&p.cls[c].tmB);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t used = 0, last_phase = 0;  // per-stage bits
      bool ok = true;
      for (int t = blockIdx.x; t < p.total_tiles && ok; t += gridDim.x) {
        const TileCoord tc = decode_tile(p, t);
        const GemmClass& k = p.cls[tc.c];
        const int nk = (k.K + kBK - 1) / kBK;
        for (int kb = 0; kb < nk; ++kb) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, s_abort, p.err, limit)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          uint8_t* a_dst = sA + stage * kATileBytes;
          uint8_t* b_dst = sB + stage * kBTileBytes;
          tma_load_3d(a_dst, &k.tmA, &full[stage], kb * kBK, tc.tm * kBM, tc.b);
          if (!k.b_mn_major) {
            tma_load_3d(b_dst, &k.tmB, &full[stage], kb * kBK, tc.tn * kBN, tc.b);
          } else {
#pragma unroll
            for (int c = 0; c < kBN / 64; ++c)
              tma_load_3d(b_dst + c * (kBK * 64 * 2), &k.tmB, &full[stage], tc.tn * kBN + c * 64, kb * kBK, tc.b);
          }
          used |= 1u << stage;
          last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Never leave the CTA with bulk copies still landing in its shared
      // memory: wait (bounded, ignoring the abort word) for the last load
      // issued into every stage.
      for (int s = 0; s < kStages; ++s)
        if ((used >> s) & 1u) wait_bounded(&full[s], (last_phase >> s) & 1u, nullptr, p.err, limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t bphase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.total_tiles && ok; t += gridDim.x) {
        const TileCoord tc = decode_tile(p, t);
        const GemmClass& k = p.cls[tc.c];
        const int nk = (k.K + kBK - 1) / kBK;
        const uint32_t idesc = p.idesc | (static_cast<uint32_t>(k.b_mn_major) << 16);
        if (!wait_bounded(&tempty[buf], bphase ^ 1u, s_abort, p.err, limit)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kBN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!wait_bounded(&full[stage], phase, s_abort, p.err, limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * kATileBytes);
          const uint32_t b_base = smem_u32(sB + stage * kBTileBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t adesc = smem_desc_sw128(a_base + kk * 32, 16, 1024);
            const uint64_t bdesc = k.b_mn_major ? smem_desc_sw128(b_base + kk * 2048, kBK * 64 * 2, 1024)
                                                : smem_desc_sw128(b_base + kk * 32, 16, 1024);
            umma_f16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[buf]);
        buf ^= 1;
        if (buf == 0) bphase ^= 1u;
      }
      // every MMA issued so far has finished before TMEM is released
      umma_commit(drain);
      wait_bounded(drain, 0, nullptr, p.err, limit);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    float* stage_buf = sEpi + (warp - 2) * kEpiWarpFloats;
    int buf = 0;
    uint32_t bphase = 0;
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x) {
      const TileCoord tc = decode_tile(p, t);
      const GemmClass& k = p.cls[tc.c];
      int ok = 1;
      if (lane == 0) ok = wait_bounded(&tfull[buf], bphase, s_abort, p.err, limit) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const int row0 = tc.tm * kBM + q * 32;
#pragma unroll 1
      for (int j = 0; j < kBN / 32; ++j) {
        const int col0 = tc.tn * kBN + j * 32;
        if (row0 >= k.M || col0 >= k.N) continue;
        if (k.symmetric && col0 < row0) continue;
        uint32_t raw[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * kBN + j * 32),
                           raw);
        tmem_wait_ld();
        float acc[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = __uint_as_float(raw[i]);
        epilogue_block(k, tc.b, row0, col0, acc, stage_buf, lane);
      }
      tc_fence_before();
      mbar_arrive(&tempty[buf]);
      buf ^= 1;
      if (buf == 0) bphase ^= 1u;
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace msb
