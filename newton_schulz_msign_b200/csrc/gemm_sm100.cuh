// gemm_sm100.cuh - persistent, warp-specialised tcgen05 GEMM engine with
// the fused epilogues of the Newton-Schulz family.
//
// One launch computes D = epilogue(A_op * B_op^T) for every tile of up to
// kMaxClasses "classes"; a class is a batch of same-shape problems whose
// operands are 3-D TMA tensors (k, row, batch).  The tile list is the
// concatenation of the classes' tiles (the host orders classes by K, longest
// first, so short tiles fill the tail of the last wave).
//
// The kernel runs on CTA pairs (clusters of two CTAs on one TPC) that share
// a tcgen05.mma.cta_group::2 instruction stream: a 256 x 256 output tile is
// one M = 256, N = 256 MMA per 16-wide K slice, with A's rows 0..127 and B's
// rows 0..127 staged in the leader CTA and the other halves in the peer.
// Each SM thus streams half of B per FLOP compared with a one-SM 128 x 256
// tile, which is what keeps the tensor pipe fed from L2.
//
// Roles inside each CTA of 2 + kEpiWarps warps (one CTA per SM, persistent
// over tiles):
//   warp 0      TMA producer, in both CTAs: loads this CTA's halves of A and
//               B (128 x 64 elements each, 128-byte swizzle) into a
//               kStages-deep ring; completion is counted on the LEADER's
//               stage barrier, which expects the bytes of both CTAs.
//   warp 1      allocates 512 TMEM columns in both CTAs (two 128 x 256 fp32
//               accumulators per CTA); in the leader it issues the MMAs and
//               tcgen05.commit-multicasts stage releases and accumulator-ready
//               signals to both CTAs.
//   warps 2..   epilogue, in both CTAs: tcgen05.ld of this CTA's 128
//               accumulator rows (warp w reads TMEM lanes 32*(w%4)..+31, two
//               warps per lane quarter, each half of the columns), fused
//               arithmetic v = alpha*acc + beta*C, then up to kMaxOuts stores,
//               each direct or transposed and each with its own gamma*I term.
//               One lane per warp then releases the accumulator on the
//               leader's barrier.
// The producer and MMA warps run their loops warp-converged and issue each
// TMA load, MMA and commit from one elected lane (see "warp-converged issue"
// in ptx_sm100.cuh).
//
// Symmetric classes ([P1] flash-muon matmul_transpose; [P3] section 4,
// triangular scheduler) enumerate only tiles (tm, tn) with tn >= tm.  A
// mirrored tile (every tile in mirror mode, the diagonal tiles otherwise)
// skips its 32x32 blocks strictly below the diagonal, stores the blocks
// above it directly and transposed into the mirrored position, and stores
// the upper part of diagonal blocks directly and their strict upper part
// transposed.  Both copies come from the same fp32 value with the same
// rounding, so the stored matrix is bit-exactly symmetric.
//
// The B operand is read K-major (rows of B_op are the output columns) or
// MN-major (B_op^T stored row-major as K x N, e.g. X in B*X), the latter via
// the UMMA descriptor's MN-major mode, so X is never transposed in memory.
//
// Symmetric intermediates (A and B of standard NS; R, Z, Q and RZ of Gram
// NS) are stored by upper 256 x 256 blocks only: a triangle-scheduled
// product writes its tiles (tm, tn >= tm) and nothing else, the diagonal
// tiles symmetrised from their upper triangle (Gram NS needs its
// intermediates exactly symmetric: products of commuting matrices such as
// Q Z are symmetric only up to rounding, and that asymmetry grows).  A
// consumer that needs rows [R, R+256) x K slice [k0, k0+64) of such a matrix
// with k0 + 64 <= R reads the stored transpose S[k0.., R..] instead and
// feeds it to the MMA through an MN-major descriptor (decided per K slice,
// identically for both CTAs of the pair).  Only the user-facing X X^T keeps
// exact mirror stores.
//
// No load anywhere uses cluster multicast: each CTA fetches its own halves.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx_sm100.cuh"

namespace msb {

constexpr int kBM = 256;      // output tile rows per CTA pair
constexpr int kHalfM = 128;   // rows per CTA (= TMEM lanes)
constexpr int kBN = 256;      // output tile columns
constexpr int kHalfN = 128;   // B rows staged per CTA
constexpr int kRowBytes = 128;  // one 128-byte swizzle row of K per operand row and stage
constexpr int kStages = 6;
// Epilogue warps per CTA: two per TMEM lane quarter, each taking half of the
// tile's columns, so that a tile's accumulator drains in half the time
// (where tiles are few, the drain of a phase's last tiles gates the next
// phase).
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;  // producer, MMA issuer, epilogue
constexpr int kATileBytes = kHalfM * kRowBytes;  // 16 KB
constexpr int kBTileBytes = kHalfN * kRowBytes;  // 16 KB

// Operand kinds: 16-bit (bf16 / fp16, kind::f16) or tf32 (fp32 words,
// kind::tf32).  A stage holds one 128-byte row of K per operand row either way.
template <bool TF32>
struct OpKind {
  static constexpr int es = TF32 ? 4 : 2;              // operand element bytes
  static constexpr int bke = kRowBytes / es;           // K elements per stage: 32 or 64
  static constexpr int kmma = TF32 ? 8 : 16;           // K per MMA instruction
  static constexpr int mn_chunk = kRowBytes / es;      // MN elements per chunk of an MN-major tile
  static constexpr int chunks = 128 / mn_chunk;        // chunks per 128 MN rows: 4 or 2
  static constexpr int chunk_bytes = bke * kRowBytes;  // 4 KB or 8 KB
  static constexpr int mn_kstep = kmma * kRowBytes;    // MN-major descriptor advance per MMA: 1024 or 2048
  // MN-major smem form: 16-bit types use the plain 128-byte swizzle (8-row
  // atoms, 1024 B); 32-bit types need the 32-byte-chunk swizzle, whose atoms
  // are 4 K rows (512 B) -- the tensor maps that feed them swizzle the same way.
  static constexpr uint32_t mn_layout = TF32 ? 1u : 2u;
  static constexpr uint32_t mn_sbo = TF32 ? 512u : 1024u;
};
constexpr int kStageBytes = kATileBytes + kBTileBytes;
// Per-warp epilogue scratch: a 32 x 32 fp32 transpose block (XOR-swizzled
// rows), or two 16-bit staging boxes of staged bulk stores.  A multiple of
// 1024 bytes from a 1024-byte aligned base, so every box is aligned to its
// swizzle pattern.
constexpr int kStageOutBytes = 32 * 32 * 4;
constexpr int kEpiBytes = kEpiWarps * kStageOutBytes;  // one scratch block per epilogue warp
constexpr int kTmemCols = 512;
constexpr int kMaxClasses = 16;
constexpr int kNumBarriers = 2 * kStages + 2 + 2 + 1;
constexpr int kSmemBytes = 1024 /* alignment slack */ + kStages * kStageBytes + kEpiBytes + kNumBarriers * 8 + 16;
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Storage types.  DT_TF32_HI / DT_TF32_LO store fp32 words: the tf32 rounding
// of v, and the tf32 rounding of the remainder v - hi (operand planes of the
// fp32-accurate path, whose products hi*hi + hi*lo + lo*hi carry ~21 bits).
enum : int { DT_BF16 = 0, DT_FP16 = 1, DT_FP32 = 2, DT_TF32_HI = 3, DT_TF32_LO = 4 };

__host__ __device__ inline int dtype_size(int dt) { return (dt == DT_BF16 || dt == DT_FP16) ? 2 : 4; }

constexpr int kMaxOuts = 4;

// One epilogue output.  Direct: D[row][col] = w; transposed: D[col][row] = w,
// where w = v + gamma * [row == col] and v = alpha*acc + beta*C.
struct EpiOut {
  void* ptr;
  long long ld, bs;  // leading dimension and batch stride, in elements
  int dtype;
  int transposed;
  float gamma;
  int blocked;  // fp32 in the 32 x 32 blocked layout (blk_off); direct stores only
  // optional, symmetric classes: the diagonal is written in fp32 to
  // diag[b * diag_bs + i] and stored as 0 in the matrix itself
  float* diag;
  long long diag_bs;
  // 16-bit row-major output written by bulk tensor stores of staged 32 x 32
  // blocks through the class's tmOut[o] (a 32 x 32 box over the stored
  // matrix, 64-byte swizzle); 0: lane-per-row stores
  int tma;
};

// One dependency of a class on an earlier class of the launch (its row-block
// counters): rows tm and/or tn of the consumer tile, or all `rows` rows,
// must have reached `target`.
constexpr int kMaxDeps = 10;
constexpr int kMaxAddends = 3;
constexpr int kTileSignals = 2 * kEpiWarps;  // arrivals per finished tile on each row it touches: a pair's epilogue warps
// DEP_EPI: waited for by the epilogue only, before it reads or stores
// anything (write-after-read orders, and the other parts of a split K)
enum : int { DEP_TM = 1, DEP_TN = 2, DEP_ALL = 4, DEP_EPI = 8 };
struct RowDep {
  const int* ptr;  // counters of batch entry 0; entry b at ptr + b * rows
  int rows, target, mode;
};

// Per-class scalars: tile schedule and epilogue (read through the constant
// cache of the kernel parameters).
struct ClassInfo {
  int M, N, K, batch;
  int tiles_m, tiles_n, tiles_per_batch, tile_begin;
  int symmetric;   // output tiles (tm, tn) with tn >= tm only
  int group;       // tile order: bands of `group` tile rows, column by column inside a band (1: row by row)
  int bn;          // tile width: 256 or 128 output columns per CTA pair (N of each MMA)
  int mirror;      // symmetric: every tile also stores its mirror (full, exactly symmetric matrix)
  int a_sym;       // A operand is a symmetric matrix stored by upper 256-blocks
  int b_sym;       // same for the B operand (K-major)
  int b_mn_major;  // B operand stored K x N (MN-major)
  int num_out, c_dtype;
  int split;       // operands are hi/lo planes (batch coordinate 2b + plane): three K passes
  long long c_plane;  // > 0: C is split too, its lo plane at C + c_plane elements
  float alpha, beta;
  const float* alpha_scale;  // optional per-batch factor on alpha
  const float* beta_scale;   // optional per-batch factor on beta
  const void* C;             // optional epilogue input, C[row][col]
  long long ldc, c_bs;
  int c_blocked;             // C is fp32 in the 32 x 32 blocked layout (blk_off)
  // optional per-row term of the C coefficient: v = alpha acc + (beta +
  // row_beta[r]) C for output row r (row_beta[b * row_beta_bs + r])
  const float* row_beta;
  long long row_beta_bs;
  // optional, symmetric classes: each epilogue warp stores the sum of v^2
  // over the tile elements it stores, the full symmetric matrix counted (an
  // element above the diagonal twice, for its unstored mirror), at
  // sumsq[b * sumsq_bs + (tm * tiles_n + tn) * kTileSignals + warp slot]
  float* sumsq;
  long long sumsq_bs;
  // split K: this class covers K slices [k_begin, k_begin + K) of the
  // product (the tensor maps span the whole K); its epilogue first adds the
  // other parts' fp32 partial tiles addend[0..num_addends) (blocked layout,
  // add_ld wide, add_bs per batch entry), in that order
  int k_begin;
  int num_addends;
  const float* addend[kMaxAddends];
  long long add_ld, add_bs;
  EpiOut out[kMaxOuts];
  // Dependencies between classes of one launch, by 256-row block of each
  // batch entry: each epilogue warp adds 1 to sig[b * tiles_m + tm] (and to
  // sig[... + tn] for an off-diagonal tile of a symmetric class) after
  // storing its rows, so a row block of a class is complete at 8 x the
  // number of its tiles that touch it.  A tile (tm, tn) starts once every
  // entry of deps[] is met (see RowDep); the epilogue acquires deps[c_dep]
  // (the producer of C) before reading C.
  RowDep deps[kMaxDeps];
  int num_deps, c_dep;
  int* sig;
};

struct alignas(64) GemmClass {
  CUtensorMap tmA;   // (k, row, batch), K-major, box 64 x 128
  CUtensorMap tmB;   // K-major: (k, col, batch) box 64 x 128; MN-major: (col, k, batch) box 64 x 64
  CUtensorMap tmA2;  // a_sym: the same matrix with a 64 x 64 box, for transposed K slices
  CUtensorMap tmB2;  // b_sym: likewise
  CUtensorMap tmOut[kMaxOuts];  // outputs with EpiOut::tma: (col, row, batch) of the stored matrix, box 32 x 32
  ClassInfo info;
};

// Dynamic tile schedule (optional): the pairs claim tiles in increasing order
// from one launch-wide counter, so a pair held up by a dependency never holds
// back work that another pair could do.  Each pair's claims are published in
// its ring of kRing entries (tag = sequence number + 1 in the high word, the
// tile in the low word); the counter and the rings start at 0.
constexpr int kRing = 16;
constexpr int kMaxSchedPairs = 128;
constexpr int kSchedBytes = 256 + kMaxSchedPairs * kRing * 8;

struct GemmParams {
  GemmClass cls[kMaxClasses];
  int num_classes;
  int total_tiles;
  uint32_t idesc;  // instruction descriptor without the B-major bit
  int* err;        // device error word (bit 0: a bounded wait ran out)
  unsigned long long timeout_ns;
  int* claim;                // dynamic schedule: next unclaimed tile (null: static round robin)
  unsigned long long* ring;  // dynamic schedule: [pair][kRing] published claims
};

static_assert(sizeof(GemmParams) <= 32764, "kernel parameter space");

struct TileCoord {
  int c, b, tm, tn;
  int tnb;  // the 256-row block of the tile's first column (= tn for 256-wide tiles)
};

// Tile order inside a class.  group = 1: row by row (the order that lets a
// chained phase start on the first finished row blocks of the one before).
// group = G > 1: bands of G tile rows; inside a band, column by column and
// top to bottom, so that the tiles a wave of CTA pairs works on at once share
// G row blocks of A and a few column blocks of B -- a working set that stays
// in L2 where the whole operand would not.  Symmetric classes keep only the
// tiles with tn >= tm: a band's first G columns form a triangle.
// Tile width of a class: a compile-time 256 in kernels built without narrow
// tiles (the common case keeps its constant-folded code), else the class's.
template <bool NARROW>
__device__ __forceinline__ int tile_bn(const ClassInfo& k) {
  return NARROW ? k.bn : kBN;
}

template <bool NARROW>
__device__ __forceinline__ TileCoord decode_tile(const GemmParams& p, int t) {
  int c = 0;
  while (c + 1 < p.num_classes && t >= p.cls[c + 1].info.tile_begin) ++c;
  const ClassInfo& k = p.cls[c].info;
  int l = t - k.tile_begin;
  int b = l / k.tiles_per_batch;
  int r = l - b * k.tiles_per_batch;
  int tm, tn;
  const int G = k.group;
  if (G <= 1) {
    if (!k.symmetric) {
      tm = r / k.tiles_n;
      tn = r - tm * k.tiles_n;
    } else {
      // tiles on or above the diagonal 256-block, row by row: row tm starts
      // at the column tile of its diagonal block
      const int per = kBM / tile_bn<NARROW>(k);
      tm = 0;
      while (true) {
        int cnt = k.tiles_n - tm * per;
        if (r < cnt) break;
        r -= cnt;
        ++tm;
      }
      tn = tm * per + r;
    }
  } else {
    int g0 = 0;
    while (true) {
      const int gh = min(G, k.tiles_m - g0);
      // tiles of the band: symmetric, a gh-row triangle then full columns
      const int tri = k.symmetric ? gh * (gh + 1) / 2 : 0;
      const int first = k.symmetric ? g0 : 0;  // first column of the band
      const int cnt = tri + gh * (k.tiles_n - first - (k.symmetric ? gh : 0));
      if (r < cnt || g0 + gh >= k.tiles_m) {
        if (r < tri) {
          int col = 0;
          while ((col + 1) * (col + 2) / 2 <= r) ++col;
          tn = first + col;
          tm = g0 + (r - col * (col + 1) / 2);
        } else {
          const int rr = r - tri;
          tn = first + (k.symmetric ? gh : 0) + rr / gh;
          tm = g0 + rr % gh;
        }
        break;
      }
      r -= cnt;
      g0 += gh;
    }
  }
  return {c, b, tm, tn, (tn * tile_bn<NARROW>(k)) / kBM};
}

// ---------------------------------------------------------------- blocked fp32 layout
//
// The fp32 copy of X is private to the library, so it is laid out for the
// epilogue's access pattern rather than row-major: 32 x 32 blocks, row-major
// over blocks, and inside a block 8 column quads of 32 rows x 4 floats.  The
// lane that owns row r of a block then finds its 4 consecutive columns next
// to those of lanes r - 1 and r + 1, so one 16-byte access per lane covers
// 512 contiguous bytes per warp.  `ldb` is the padded column count (a
// multiple of 32); a matrix occupies round_up(rows, 32) x ldb floats.
__host__ __device__ __forceinline__ long long blk_off(long long r, long long c, long long ldb) {
  return (((r >> 5) * (ldb >> 5) + (c >> 5)) << 10) + (((c & 31) >> 2) << 7) + ((r & 31) << 2) + (c & 3);
}

// ---------------------------------------------------------------- row I/O

__device__ __forceinline__ float load_elem(const char* p, int dt) {
  if (dt == DT_FP32 || dt == DT_TF32_HI || dt == DT_TF32_LO) return *reinterpret_cast<const float*>(p);
  if (dt == DT_BF16) return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
  return __half2float(*reinterpret_cast<const __half*>(p));
}

__device__ __forceinline__ float split_value(int dt, float v) {
  if (dt == DT_TF32_HI) return to_tf32(v);
  if (dt == DT_TF32_LO) return to_tf32(v - to_tf32(v));
  return v;
}

__device__ __forceinline__ void store_elem(char* p, int dt, float v) {
  if (dt == DT_FP32 || dt == DT_TF32_HI || dt == DT_TF32_LO)
    *reinterpret_cast<float*>(p) = split_value(dt, v);
  else if (dt == DT_BF16)
    *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(v);
  else
    *reinterpret_cast<__half*>(p) = __float2half_rn(v);
}

// Loads 32 consecutive elements of one row; lanes outside `mask` read 0.
__device__ __forceinline__ void load_row32(const char* rowp, int dt, uint32_t mask, float (&v)[32]) {
  const int es = dtype_size(dt);
  if (mask == 0xFFFFFFFFu && (reinterpret_cast<uintptr_t>(rowp) & 15) == 0) {
    if (dtype_size(dt) == 4) {
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
    if (dt == DT_FP32 || dt == DT_TF32_HI || dt == DT_TF32_LO) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        reinterpret_cast<float4*>(rowp)[i] =
            make_float4(split_value(dt, v[4 * i]), split_value(dt, v[4 * i + 1]), split_value(dt, v[4 * i + 2]),
                        split_value(dt, v[4 * i + 3]));
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
//
// Each lane owns one accumulator row (TMEM lane = tile row) and moves its 32
// consecutive elements of a block with 16-byte accesses.  Transposed outputs
// go through a 32 x 32 fp32 scratch block in shared memory whose rows are
// padded to 33 words, so that writing by rows and reading by columns are both
// conflict-free with one instruction per access.

__device__ __forceinline__ char* gaddr(const void* p, int dt, long long ld, long long bs, int b, long long r,
                                       long long c) {
  return const_cast<char*>(reinterpret_cast<const char*>(p)) +
         (static_cast<long long>(b) * bs + r * ld + c) * dtype_size(dt);
}

__device__ __forceinline__ uint32_t lane_mask(int n) { return n >= 32 ? 0xFFFFFFFFu : ((1u << n) - 1u); }

// Epilogue input of the block at (row0, col0) for this lane's row.
__device__ __forceinline__ void load_c(const ClassInfo& k, int b, int row0, int col0, int lane, float (&cv)[32]) {
  const int r = row0 + lane;
  if (k.c_blocked) {
    // whole padded block, coalesced; elements outside C read as 0
    const float* q = reinterpret_cast<const float*>(k.C) + static_cast<long long>(b) * k.c_bs +
                     blk_off(row0, col0, k.ldc) + 4 * lane;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 f = *reinterpret_cast<const float4*>(q + 128 * j);
      cv[4 * j + 0] = f.x, cv[4 * j + 1] = f.y, cv[4 * j + 2] = f.z, cv[4 * j + 3] = f.w;
    }
    if (r >= k.M || col0 + 32 > k.N) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (r >= k.M || col0 + i >= k.N) cv[i] = 0.0f;
    }
    return;
  }
  const uint32_t m = (r < k.M) ? lane_mask(k.N - col0) : 0u;
  const char* hp = gaddr(k.C, k.c_dtype, k.ldc, k.c_bs, b, r, col0);
  load_row32(hp, k.c_dtype, m, cv);
  if (k.c_plane > 0) {  // split C: value = hi + lo
    float lo[32];
    load_row32(hp + k.c_plane * 4, DT_FP32, m, lo);
#pragma unroll
    for (int i = 0; i < 32; ++i) cv[i] += lo[i];
  }
}

// ---------------------------------------------------------------- staged bulk stores
//
// A 16-bit output block leaves through a 32 x 32 staging box in the warp's
// scratch, which lane 0 hands to a bulk tensor store: whole lines reach L2
// instead of one 16-byte piece of 32 different rows per store instruction.
// The box has 64-byte rows in the tensor map's 64-byte swizzle: 16-byte
// piece i of row r sits at piece i ^ ((r >> 1) & 3) of the row, so when lane
// l writes piece i of its row l, each group of 8 lanes covers the 8 16-byte
// bank groups of a 128-byte line (one wavefront per group).  A transposed
// box is read out of the first by columns: lane l loads column l, 32
// two-byte loads that each stay inside one 64-byte row.
constexpr int kBoxBytes = 32 * 32 * 2;
static_assert(2 * kBoxBytes <= kStageOutBytes, "two staging boxes per epilogue warp");

__device__ __forceinline__ void pack16(const float (&w)[32], int dt, uint32_t (&h)[16]) {
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    if (dt == DT_BF16) {
      __nv_bfloat162 v = __floats2bfloat162_rn(w[2 * m], w[2 * m + 1]);
      h[m] = *reinterpret_cast<uint32_t*>(&v);
    } else {
      __half2 v = __floats2half2_rn(w[2 * m], w[2 * m + 1]);
      h[m] = *reinterpret_cast<uint32_t*>(&v);
    }
  }
}

__device__ __forceinline__ void stage_row(uint8_t* box, int lane, const uint32_t (&h)[16]) {
  uint8_t* rowp = box + lane * 64;
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<uint4*>(rowp + 16 * (i ^ sw)) = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
}

// Column `lane` of a staged box, packed like a row: element j of the result
// is box[j][lane].
__device__ __forceinline__ void stage_col(const uint8_t* box, int lane, uint32_t (&h)[16]) {
  const int piece = lane >> 3, within = 2 * (lane & 7);
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const int r0 = 2 * m, r1 = 2 * m + 1;
    const uint32_t lo = *reinterpret_cast<const uint16_t*>(box + r0 * 64 + 16 * (piece ^ ((r0 >> 1) & 3)) + within);
    const uint32_t hi = *reinterpret_cast<const uint16_t*>(box + r1 * 64 + 16 * (piece ^ ((r1 >> 1) & 3)) + within);
    h[m] = lo | (hi << 16);
  }
}

// One 32x32 block: this lane owns output row `row0 + lane`, columns
// col0..col0+31, whose fp32 accumulators are in `acc` and epilogue input in
// `cv` (when the class has one).  `mirror`: the block is stored together
// with its transpose at the mirrored position (symmetric classes: every
// block of mirror classes, and the blocks of diagonal tiles); on a diagonal
// block the upper part and its mirror fill the block, so the stored matrix
// is exactly symmetric there.
// alpha and beta: the class's coefficients with their per-batch scales and
// this lane's row term applied (formed once per tile).
__device__ __forceinline__ void epilogue_block(const ClassInfo& k, const CUtensorMap* tmo, int b, int row0, int col0,
                                               bool mirror, float (&acc)[32], const float (&cv)[32], float alpha,
                                               float beta, float* scratch, int lane, float& sq) {
  const int r = row0 + lane;
  const bool diag = mirror && (col0 == row0);
  const uint32_t colmask = lane_mask(k.N - col0);
  const uint32_t rowmask = lane_mask(k.M - row0);

  if (k.C != nullptr) {
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = fmaf(alpha, acc[i], beta * cv[i]);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] *= alpha;
  }
  if (k.sumsq != nullptr && r < k.M) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int c = col0 + i;
      const float wgt = c > r ? 2.0f : (c == r ? 1.0f : 0.0f);
      if (c < k.N) sq = fmaf(wgt * acc[i], acc[i], sq);
    }
  }

#pragma unroll 1
  for (int o = 0; o < k.num_out; ++o) {
    const EpiOut& e = k.out[o];
    float w[32];
    const float g = (col0 == row0) ? e.gamma : 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i] = (i == lane) ? acc[i] + g : acc[i];
    if (e.diag != nullptr && col0 == row0) {
      // this lane's diagonal element (r, r) goes to the fp32 vector
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i == lane) {
          if (r < k.M) e.diag[static_cast<long long>(b) * e.diag_bs + r] = w[i];
          w[i] = 0.0f;
        }
    }
    if (e.blocked) {
      // whole padded block, coalesced (elements outside the matrix are 0)
      float* q = reinterpret_cast<float*>(e.ptr) + static_cast<long long>(b) * e.bs + blk_off(row0, col0, e.ld) + 4 * lane;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float4*>(q + 128 * j) = make_float4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
      continue;
    }
    const bool direct = !e.transposed;
    const bool trans = e.transposed || mirror;
    if (e.tma) {
      // staged: box 0 holds the block, box 1 its transpose (or, on a diagonal
      // block, the exactly symmetric block: the upper part and its mirror)
      uint8_t* s0 = reinterpret_cast<uint8_t*>(scratch);
      uint8_t* s1 = s0 + kBoxBytes;
      if (lane == 0) bulk_wait_read_all();  // the previous stores have read both boxes
      __syncwarp();
      uint32_t h[16];
      pack16(w, e.dtype, h);
      stage_row(s0, lane, h);
      if (trans) {
        __syncwarp();
        uint32_t t[16];
        stage_col(s0, lane, t);
        if (diag) {
          // columns c < r take the mirror's value (row c, column r)
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            const uint32_t lo = (2 * m < lane) ? (t[m] & 0xFFFFu) : (h[m] & 0xFFFFu);
            const uint32_t hi = (2 * m + 1 < lane) ? (t[m] & 0xFFFF0000u) : (h[m] & 0xFFFF0000u);
            t[m] = lo | hi;
          }
        }
        stage_row(s1, lane, t);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const void* tm = tmo + o;
        if (diag) {
          tma_store_3d(tm, s1, col0, row0, b);
        } else {
          if (direct) tma_store_3d(tm, s0, col0, row0, b);
          if (trans) tma_store_3d(tm, s1, row0, col0, b);
        }
        bulk_commit_group();
      }
      continue;
    }
    if (direct && r < k.M) {
      uint32_t m = colmask;
      if (diag) m &= (0xFFFFFFFFu << lane);  // columns c >= r; the mirror supplies c < r
      store_row32(gaddr(e.ptr, e.dtype, e.ld, e.bs, b, r, col0), e.dtype, m, w);
    }
    if (trans) {
      // scratch[i][lane] = w(row0 + lane, col0 + i), word lane ^ i of row i
      // (conflict-free both ways); lane l then reads its column l, which is
      // row col0 + l of the transposed block
      if (lane == 0) bulk_wait_read_all();  // staged stores of an earlier output have read the scratch
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 32; ++i) scratch[i * 32 + (lane ^ i)] = w[i];
      __syncwarp();
      // w now takes the transposed block's row
#pragma unroll
      for (int j = 0; j < 32; ++j) w[j] = scratch[lane * 32 + (j ^ lane)];
      __syncwarp();
      const int tr = col0 + lane;  // row of the transposed block
      if (tr < k.N) {
        uint32_t m = rowmask;
        if (diag) m &= (lane == 0) ? 0u : (0xFFFFFFFFu >> (32 - lane));  // rows r < c (strict)
        store_row32(gaddr(e.ptr, e.dtype, e.ld, e.bs, b, tr, row0), e.dtype, m, w);
      }
    }
  }
}

// ---------------------------------------------------------------- tile sequence
//
// The seq-th tile of a pair.  Static: pair + seq * num_pairs.  Dynamic: the
// claimer (the leader CTA's producer) takes the next tile from the counter
// when it is ready to load it, and publishes it; every other role of the
// pair (the peer's producer, the MMA issuer, both epilogues) reads the
// publication.  A tile index >= total_tiles ends every role's loop.  Tiles
// are claimed in increasing order and every dependency points to a lower
// index, so the lowest unfinished tile always belongs to a pair that is
// working on it.  The claimer runs at most a few tiles ahead of the pair's
// last reader (the epilogue, held back by two TMEM buffers and the operand
// stages), well inside the ring.  (Claiming one tile ahead was measured: it
// hides the publication latency but holds ready tiles on busy pairs, which
// costs more wherever dependencies gate the schedule.)
__device__ __forceinline__ bool next_tile(const GemmParams& p, int pair, int num_pairs, bool claimer, int seq,
                                          volatile int* abort_word, uint64_t limit_ns, int* t_out) {
  if (p.claim == nullptr) {
    *t_out = pair + seq * num_pairs;
    return true;
  }
  unsigned long long* slot = p.ring + pair * kRing + (seq % kRing);
  const unsigned long long tag = static_cast<unsigned long long>(seq + 1);
  if (claimer) {
    const int t = atomicAdd(p.claim, 1);
    st_release_gpu_u64(slot, (tag << 32) | static_cast<unsigned int>(t));
    *t_out = t;
    return true;
  }
  unsigned long long v = ld_acquire_gpu_u64(slot);
  if ((v >> 32) != tag) {
    const uint64_t t0 = globaltimer_ns();
    while (true) {
      __nanosleep(32);
      v = ld_acquire_gpu_u64(slot);
      if ((v >> 32) == tag) break;
      if (abort_word != nullptr && *abort_word) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        if (abort_word != nullptr) *abort_word = 1;
        if (p.err != nullptr) atomicOr(p.err, 1);
        return false;
      }
    }
  }
  *t_out = static_cast<int>(v & 0xFFFFFFFFu);
  return true;
}

// ---------------------------------------------------------------- kernel

// Launched with clusters of 2 CTAs along x; gridDim.x is even.  TF32 selects
// the operand kind (see OpKind).
template <bool TF32, bool NARROW>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_sm100_kernel(const __grid_constant__ GemmParams p) {
  using OK = OpKind<TF32>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kATileBytes;
  uint8_t* sOut = sB + kStages * kBTileBytes;  // epilogue staging, kEpiBytes
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + kEpiBytes);
  uint64_t* full = bars;             // leader: both CTAs' loads of a stage landed
  uint64_t* empty = bars + kStages;  // both: the MMAs reading a stage finished
  uint64_t* tfull = bars + 2 * kStages;  // both: accumulator buffer ready
  uint64_t* tempty = tfull + 2;          // leader: both epilogues drained a buffer
  uint64_t* drain = tempty + 2;          // leader: every issued MMA finished
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + kNumBarriers);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
  const uint64_t limit = p.timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * kEpiWarps);  // one arrival per epilogue warp of each CTA
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(s_tmem, kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    for (int c = 0; c < p.num_classes; ++c) {
      tma_prefetch_desc(&p.cls[c].tmA);
      tma_prefetch_desc(&p.cls[c].tmB);
    }
  }
  tc_fence_before();
  __syncthreads();
  // both CTAs' barriers are initialised before either signals the other's
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  // Launched as a programmatic dependent of the previous kernel on the
  // stream: the set-up above overlaps that kernel's tail, and nothing below
  // touches global memory before it has completed.  (Without the launch
  // attribute the wait returns at once.)
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    // The whole warp runs the loop (see "warp-converged issue" in
    // ptx_sm100.cuh): lane 0 claims tiles and broadcasts them, every lane
    // waits on the barriers and counters (so that each has its own acquire),
    // and one elected lane issues each load.
    {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t used = 0, last_phase = 0;  // per-stage bits (leader only)
      bool ok = true;
      for (int seq = 0; ok; ++seq) {
        int t = 0, got = 1;
        if (lane == 0) got = next_tile(p, pair, num_pairs, leader, seq, s_abort, limit, &t) ? 1 : 0;
        got = __shfl_sync(0xFFFFFFFFu, got, 0);
        t = __shfl_sync(0xFFFFFFFFu, t, 0);
        if (!got) {
          ok = false;
          break;
        }
        if (t >= p.total_tiles) break;
        const TileCoord tc = decode_tile<NARROW>(p, t);
        const ClassInfo& k = p.cls[tc.c].info;
        // per-tile state in registers
        const int nk = (k.K + OK::bke - 1) / OK::bke;
        const int passes = k.split ? 3 : 1;  // split: hi*hi, hi*lo, lo*hi per K slice
        const int arow = tc.tm * kBM + static_cast<int>(rank) * kHalfM;
        const int bn = tile_bn<NARROW>(k);
        const int bhalf = bn / 2;  // B rows (output columns) staged per CTA
        const int bcol = tc.tn * bn + static_cast<int>(rank) * bhalf;
        const int bch = bhalf / OK::mn_chunk;  // MN-major chunks of B per CTA
        const uint32_t stage_tx = 2u * static_cast<uint32_t>(kATileBytes + bhalf * kRowBytes);  // both CTAs
        const int ko = k.k_begin / OK::bke;  // first K slice of this class (split K)
        const int a_tr = k.a_sym ? (tc.tm * kBM) / OK::bke - ko : 0;  // K slices below this read A transposed
        // (B is stored by upper 256-blocks: the K slices below the 256-block of
        // the tile's columns are read from the stored transpose)
        const int b_tr = k.b_sym ? (tc.tnb * kBM) / OK::bke - ko : 0;
        const bool b_mn = k.b_mn_major != 0;
        const GemmClass& g = p.cls[tc.c];
        const void* tmA = &g.tmA;
        const void* tmA2 = &g.tmA2;
        const void* tmB = &g.tmB;
        const void* tmB2 = &g.tmB2;
        if (k.num_deps > 0) {
          // operands produced earlier in this launch (and earlier readers of
          // the buffers this tile overwrites): wait for their row blocks.
          // Every lane waits, so the elected lane that issues the loads has
          // its own acquire.
          bool dok = true;
          for (int e = 0; e < k.num_deps && dok; ++e) {
            const RowDep& d = k.deps[e];
            if (d.mode & DEP_EPI) continue;
            const int* base = d.ptr + static_cast<long long>(tc.b) * d.rows;
            if (d.mode & DEP_ALL) {
              for (int r = 0; r < d.rows && dok; ++r) dok = wait_counter(base + r, d.target, s_abort, p.err, limit);
            } else {
              if (d.mode & DEP_TM) dok = dok && wait_counter(base + tc.tm, d.target, s_abort, p.err, limit);
              if (d.mode & DEP_TN) dok = dok && wait_counter(base + tc.tnb, d.target, s_abort, p.err, limit);
            }
          }
          if (!__all_sync(0xFFFFFFFFu, dok)) {
            ok = false;
            break;
          }
          fence_proxy_async_global();
        }
        for (int step = 0; step < nk * passes; ++step) {
          const int kb = step / passes, pass = step - kb * passes;
          const int za = passes == 1 ? tc.b : 2 * tc.b + (pass == 2 ? 1 : 0);
          const int zb = passes == 1 ? tc.b : 2 * tc.b + (pass == 1 ? 1 : 0);
          if (!__all_sync(0xFFFFFFFFu, wait_bounded(&empty[stage], phase ^ 1u, s_abort, p.err, limit))) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx_w(&full[stage], stage_tx);
          const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
          uint8_t* a_dst = sA + stage * kATileBytes;
          uint8_t* b_dst = sB + stage * kBTileBytes;
          const int k0 = (kb + ko) * OK::bke;
          if (kb < a_tr) {
            // stored transpose: rows k0.. of S, columns arow..arow+127 (MN-major)
#pragma unroll
            for (int c = 0; c < OK::chunks; ++c)
              tma_load_3d_pair_w(a_dst + c * OK::chunk_bytes, tmA2, fbar, arow + c * OK::mn_chunk, k0, za);
          } else {
            tma_load_3d_pair_w(a_dst, tmA, fbar, k0, arow, za);
          }
          if (kb < b_tr || b_mn) {
            const void* tm = (kb < b_tr) ? tmB2 : tmB;
#pragma unroll
            for (int c = 0; c < OK::chunks; ++c)
              if (c < bch) tma_load_3d_pair_w(b_dst + c * OK::chunk_bytes, tm, fbar, bcol + c * OK::mn_chunk, k0, zb);
          } else {
            tma_load_3d_pair_w(b_dst, tmB, fbar, k0, bcol, zb);
          }
          used |= 1u << stage;
          last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Never leave the pair with bulk copies still landing: the leader's
      // stage barriers count both CTAs' bytes, so the leader waits (bounded,
      // ignoring the abort word) for the last phase issued into each stage.
      if (leader && lane == 0)
        for (int s = 0; s < kStages; ++s)
          if ((used >> s) & 1u) wait_bounded(&full[s], (last_phase >> s) & 1u, nullptr, p.err, limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    // The whole warp runs the loop; every lane waits, one elected lane issues
    // each MMA and commit (see "warp-converged issue" in ptx_sm100.cuh).
    if (leader) {
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t bphase = 0;
      bool ok = true;
      const uint32_t idesc0 = p.idesc;
      const uint32_t sA0 = smem_u32(sA), sB0 = smem_u32(sB);
      // K-major and MN-major descriptors of stage 0; stage s adds s * tile
      // bytes and K step kk adds 32 (K-major) or 2048 (MN-major) bytes, all
      // in the 16-byte-unit start-address field.
      const uint64_t dA_k = smem_desc_sw128(sA0, 16, 1024), dA_mn = smem_desc_sw128(sA0, OK::chunk_bytes, OK::mn_sbo, OK::mn_layout);
      const uint64_t dB_k = smem_desc_sw128(sB0, 16, 1024), dB_mn = smem_desc_sw128(sB0, OK::chunk_bytes, OK::mn_sbo, OK::mn_layout);
      for (int seq = 0; ok; ++seq) {
        int t = 0, got = 1;
        if (lane == 0) got = next_tile(p, pair, num_pairs, false, seq, s_abort, limit, &t) ? 1 : 0;
        got = __shfl_sync(0xFFFFFFFFu, got, 0);
        t = __shfl_sync(0xFFFFFFFFu, t, 0);
        if (!got || t >= p.total_tiles) break;
        const TileCoord tc = decode_tile<NARROW>(p, t);
        const ClassInfo& k = p.cls[tc.c].info;
        const int nk = (k.K + OK::bke - 1) / OK::bke;
        const int passes = k.split ? 3 : 1;
        const int ko = k.k_begin / OK::bke;
        const int a_tr = k.a_sym ? (tc.tm * kBM) / OK::bke - ko : 0;
        const int b_tr = k.b_sym ? (tc.tnb * kBM) / OK::bke - ko : (k.b_mn_major ? nk : 0);
        // the MMA's N is the class's tile width
        const uint32_t idesc_n =
            NARROW ? (idesc0 & ~(0x3Fu << 17)) | (static_cast<uint32_t>(k.bn >> 3) << 17) : idesc0;
        if (!__all_sync(0xFFFFFFFFu, wait_bounded(&tempty[buf], bphase ^ 1u, s_abort, p.err, limit))) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kBN);
        for (int step = 0; step < nk * passes; ++step) {
          const int kb = step / passes;
          if (!__all_sync(0xFFFFFFFFu, wait_bounded(&full[stage], phase, s_abort, p.err, limit))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const bool a_mn = kb < a_tr;
          const bool b_mn = kb < b_tr;
          const uint32_t idesc = idesc_n | (static_cast<uint32_t>(a_mn) << 15) | (static_cast<uint32_t>(b_mn) << 16);
          const uint64_t da = (a_mn ? dA_mn : dA_k) + static_cast<uint64_t>((stage * kATileBytes) >> 4);
          const uint64_t db = (b_mn ? dB_mn : dB_k) + static_cast<uint64_t>((stage * kBTileBytes) >> 4);
          const uint32_t sa = a_mn ? (OK::mn_kstep >> 4) : (32 >> 4);
          const uint32_t sb = b_mn ? (OK::mn_kstep >> 4) : (32 >> 4);
#pragma unroll
          for (int kk = 0; kk < OK::bke / OK::kmma; ++kk) {
            const uint32_t acc = (step | kk) != 0 ? 1u : 0u;
            if (TF32)
              umma_tf32_pair_w(d_tmem, da + kk * sa, db + kk * sb, idesc, acc);
            else
              umma_f16_pair_w(d_tmem, da + kk * sa, db + kk * sb, idesc, acc);
          }
          umma_commit_pair_mc_w(&empty[stage], 0x3);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair_mc_w(&tfull[buf], 0x3);
        buf ^= 1;
        if (buf == 0) bphase ^= 1u;
      }
      // every MMA issued so far has finished before TMEM is released
      umma_commit_pair_mc_w(drain, 0x1);
      if (lane == 0) wait_bounded(drain, 0, nullptr, p.err, limit);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    const int ew = warp - 2;  // epilogue warp index
    float* scratch = reinterpret_cast<float*>(sOut + ew * kStageOutBytes);
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[1]), 0);
    int buf = 0;
    uint32_t bphase = 0;
    for (int seq = 0;; ++seq) {
      int t = 0, got = 1;
      if (lane == 0) got = next_tile(p, pair, num_pairs, false, seq, s_abort, limit, &t) ? 1 : 0;
      got = __shfl_sync(0xFFFFFFFFu, got, 0);
      t = __shfl_sync(0xFFFFFFFFu, t, 0);
      if (!got || t >= p.total_tiles) break;
      const TileCoord tc = decode_tile<NARROW>(p, t);
      const ClassInfo& k = p.cls[tc.c].info;
      const int row0 = tc.tm * kBM + static_cast<int>(rank) * kHalfM + q * 32;
      // this warp's 32-column blocks of the tile: [jbeg, jend) (two warps per
      // TMEM lane quarter, each half of the tile's columns)
      const int bn = tile_bn<NARROW>(k);
      const int bpw = (bn / 32) / (kEpiWarps / 4);
      const int jbeg = (ew >> 2) * bpw, jend = jbeg + bpw;
      const int coln = tc.tn * bn;  // the tile's first column
      // mirrored tiles (every tile of a mirror class, and the tiles inside a
      // diagonal 256-block) visit only blocks on or above the diagonal
      const bool mirror = k.symmetric && (k.mirror || tc.tm == tc.tnb);
      int jfirst = jbeg;
      if (mirror)
        while (jfirst < jend && coln + jfirst * 32 < row0) ++jfirst;
      const bool has_c = k.C != nullptr;
      int ok = 1;
      if (has_c && k.c_dep >= 0) {
        // C was written earlier in this launch: acquire it for this warp
        const RowDep& dd = k.deps[k.c_dep];
        const int* d = dd.ptr + static_cast<long long>(tc.b) * dd.rows + tc.tm;
        if (lane == 0) ok = wait_counter(d, dd.target, s_abort, p.err, limit) ? 1 : 0;
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) break;
        // each lane's own acquire orders its C loads (plain, L1-cached)
        // after the producers' release
        (void)ld_acquire_gpu(d);
      }
      {
        // epilogue-only dependencies (the other parts of a split K, whose
        // partials are added below, and write-after-read orders: nothing is
        // stored before they are met); every lane waits, so every lane has
        // its own acquire
        bool eok = true;
        for (int e = 0; e < k.num_deps && eok; ++e) {
          const RowDep& d = k.deps[e];
          if (!(d.mode & DEP_EPI)) continue;
          const int* base = d.ptr + static_cast<long long>(tc.b) * d.rows;
          if (d.mode & DEP_ALL) {
            for (int r = 0; r < d.rows && eok; ++r) eok = wait_counter(base + r, d.target, s_abort, p.err, limit);
          } else {
            if (d.mode & DEP_TM) eok = eok && wait_counter(base + tc.tm, d.target, s_abort, p.err, limit);
            if (d.mode & DEP_TN) eok = eok && wait_counter(base + tc.tnb, d.target, s_abort, p.err, limit);
          }
        }
        if (!__all_sync(0xFFFFFFFFu, eok)) break;
      }
      // the first block's epilogue input is read before the accumulator is
      // ready, each next block's just before its accumulator load
      float cv[32];
      float sq = 0.0f;  // this lane's part of the tile's sum of squares (sumsq classes)
      if (has_c && row0 < k.M && jfirst < jend && coln + jfirst * 32 < k.N)
        load_c(k, tc.b, row0, coln + jfirst * 32, lane, cv);
      // the epilogue coefficients of this lane's row, for every block of the tile
      float alpha = k.alpha, beta = k.beta;
      if (k.row_beta != nullptr && row0 + lane < k.M)
        beta += k.row_beta[static_cast<long long>(tc.b) * k.row_beta_bs + row0 + lane];
      if (k.alpha_scale != nullptr) alpha *= k.alpha_scale[tc.b];
      if (k.beta_scale != nullptr) beta *= k.beta_scale[tc.b];
      if (lane == 0) ok = wait_bounded(&tfull[buf], bphase, s_abort, p.err, limit) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int j = jfirst; j < jend; ++j) {
        const int col0 = coln + j * 32;
        if (row0 >= k.M || col0 >= k.N) break;
        // (issued before the accumulator load, so that the two overlap)
        if (has_c && j > jfirst) load_c(k, tc.b, row0, col0, lane, cv);
        uint32_t raw[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * kBN + j * 32),
                           raw);
        tmem_wait_ld();
        float acc[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = __uint_as_float(raw[i]);
        for (int a = 0; a < k.num_addends; ++a) {
          // split K: this block of another part's fp32 partial (coalesced)
          const float* ap = k.addend[a] + static_cast<long long>(tc.b) * k.add_bs + blk_off(row0, col0, k.add_ld) + 4 * lane;
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4) {
            const float4 f = *reinterpret_cast<const float4*>(ap + 128 * j4);
            acc[4 * j4 + 0] += f.x;
            acc[4 * j4 + 1] += f.y;
            acc[4 * j4 + 2] += f.z;
            acc[4 * j4 + 3] += f.w;
          }
        }
        epilogue_block(k, p.cls[tc.c].tmOut, tc.b, row0, col0, mirror, acc, cv, alpha, beta, scratch, lane, sq);
      }
      if (k.sumsq != nullptr) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xFFFFFFFFu, sq, o);
        if (lane == 0)
          k.sumsq[static_cast<long long>(tc.b) * k.sumsq_bs + (static_cast<long long>(tc.tm) * k.tiles_n + tc.tn) * kTileSignals +
                  rank * kEpiWarps + ew] = sq;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(buf ? tempty_leader1 : tempty_leader0);
      if (k.sig != nullptr) {
        // publish this warp's rows of the tile to later classes of the launch
        // (lane 0's staged stores complete first).  Every lane orders its
        // generic stores before later async-proxy reads; the warp barrier
        // orders all lanes' stores before lane 0's release, which is
        // cumulative, so no lane needs a gpu-scope fence of its own
        // (measured: one such fence per tile cost 1-2.5% on chains of small
        // products)
        if (lane == 0) bulk_wait_all();
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) {
          int* sg = k.sig + static_cast<long long>(tc.b) * k.tiles_m;
          red_release_gpu_add(sg + tc.tm, 1);
          if (k.symmetric && tc.tnb != tc.tm) red_release_gpu_add(sg + tc.tnb, 1);
        }
      }
      buf ^= 1;
      if (buf == 0) bphase ^= 1u;
    }
    // the staging boxes stay in use until the last stores have completed
    if (lane == 0) bulk_wait_all();
  }

  // Reconverge every warp first: in the producer and MMA warps only lane 0
  // ran the role loop, and a block barrier reached by a warp in two pieces
  // would let the CTA go on (and release TMEM) while others still work.
  __syncwarp();
  __syncthreads();
  // no CTA of the pair leaves while the other may still signal it
  cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace msb
