// Grouped GEMM on the 5th-generation tensor cores (sm_100a: tcgen05.mma with
// TMEM accumulators, operands staged by TMA), one launch per wave.
//
// Every node g of a wave multiplies its own activations A_g [M x K] by the
// weights of its own layer B_l [N x K]^T (skill page "Diagonal Batching for
// Recurrent Memory Transformers", "GroupedGEMM Operations": the wave's layers
// batched in one grouped kernel; Pith review of arXiv 2506.05229, "What
// carries the argument": stacked weights + grouped matrix multiplication).
// The stacked weights are one 3-D tensor [L, N, K]; the layer index is the
// outer TMA coordinate, so a tile of node g loads B with coordinate l(g).
//
// Operands are 16-bit, both fp16 or both bf16 (a runtime instruction-
// descriptor field), or both fp32 multiplied at tf32 precision (kind::tf32,
// a template variant: 32 fp32 words fill the same 128-byte swizzle row as 64
// 16-bit values, and one K = 8 instruction covers the same 32 bytes as one
// K = 16 instruction of kind::f16, so the shared-memory layout, descriptors
// and pipeline are identical).
//
// Kernel structure (persistent, one CTA per SM, 320 threads):
//   warp 0      TMA producer: A tile 128x64 and B tile BNx64 (16-bit, 128-byte
//               swizzle) per pipeline stage
//   warp 1      allocates TMEM; one lane issues tcgen05.mma (M=128, N=BN,
//               K=16) and commits stage/accumulator barriers
//   warps 2..9  epilogue: tcgen05.ld of the accumulator rows (thread = row;
//               warps w and w+4 share TMEM lanes 32*(w%4).. and split the
//               tile's columns in halves), fused epilogue, global stores
// Two TMEM accumulators (2 x BN columns) let the epilogue of tile t overlap
// the main loop of tile t+1.  Tiles never straddle nodes: a node's rows are
// the middle TMA coordinate with extent M, rows past M read as zeros.
//
// Ragged last row tile (swap_tail).  When a node's last row tile holds at
// most SWAP_ROWS rows (1040 = 8 x 128 + 16 at 1B), it is computed transposed:
// D^T = B_tile A_rows^T with the weight rows as the 128-row operand and the
// SWAP_ROWS activation rows as N, one M = 128, N = SWAP_ROWS instruction per
// 128 weight rows and K step, instead of a 128 x BN product of which 7/8 are
// padding.  The epilogue warps move D^T through shared memory (a row per
// activation row) and the warps of TMEM quarter 0 run the ordinary epilogue
// on those rows.
//
// 16-bit outputs (the next GEMM's operand copy, SwiGLU and QKV results) are
// written through a 2 KB shared-memory slot per epilogue warp: a lane owns a
// row, so a direct 16-byte store instruction touches 32 rows; through the
// slot (16-byte pieces XOR-swizzled by row, conflict-free both ways) every
// store instruction writes whole 64-byte row pieces of 8 rows.
// Every mbarrier wait is bounded (about one second); on timeout the kernel
// sets the device error word, drains its own outstanding copies and MMAs,
// frees TMEM and returns.
#include <cstdlib>
#include <type_traits>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "armt_internal.cuh"
#include "tc_gemm.cuh"
#include "tcgen05_ptx.cuh"

namespace armt {

namespace {

using namespace tc;

constexpr int BM = 128;
constexpr int BK = 64;                 // 64 bf16 = 128 bytes = one swizzle row
constexpr int EPI_WARPS = 8;           // two warps per TMEM lane quarter, each half of the columns
constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
constexpr int SWAP_ROWS = 16;          // transposed ragged tile: rows (= MMA N) it covers
constexpr int XS_SLOT = 2048;          // per epilogue warp: 32 rows x 64 bytes of 16-bit output

__device__ __forceinline__ void store_f16x32(f16* dst, const float* v) {
  // 32 values = 64 bytes: four 16-byte stores (dst 16-byte aligned)
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 pk;
    uint32_t* w = reinterpret_cast<uint32_t*>(&pk);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h2 = __floats2half2_rn(v[q * 8 + 2 * i], v[q * 8 + 2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h2);
    }
    reinterpret_cast<uint4*>(dst)[q] = pk;
  }
}

template <int BN>
struct Smem {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN >= 256 ? 4 : (BN >= 128 ? 6 : 8);
  static constexpr int BAR_OFFSET = STAGES * STAGE_BYTES;
  // transposed ragged tile (BN a multiple of 128): A box of SWAP_ROWS rows and
  // the staging area of D^T, one row of BN (+4 against bank conflicts) fp32
  // per activation row
  static constexpr bool SWAP = BN % 128 == 0;
  static constexpr int SWAP_A_BYTES = SWAP_ROWS * BK * 2;
  static constexpr int STG_PITCH = BN + 4;
  static constexpr int STG_OFFSET = BAR_OFFSET + 256;
  static constexpr int STG_BYTES = SWAP ? SWAP_ROWS * STG_PITCH * 4 : 0;
  static constexpr int XS_OFFSET = STG_OFFSET + STG_BYTES;      // 16-byte aligned
  static constexpr int TOTAL = XS_OFFSET + EPI_WARPS * XS_SLOT + 1024;   // + alignment slack
  static_assert(TOTAL + 64 <= 227 * 1024, "shared memory per CTA");
};

__device__ __forceinline__ void store_f32x32(float* dst, const float* v, int valid_cols) {
  if (valid_cols >= 32 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
      reinterpret_cast<float4*>(dst)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < valid_cols) dst[i] = v[i];
  }
}

__device__ __forceinline__ void store_act32(f16* dst, const float* v, int valid_cols) {
  if (valid_cols >= 32 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
    store_f16x32(dst, v);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < valid_cols) dst[i] = __float2half_rn(v[i]);
  }
}

__device__ __forceinline__ void store_bf16_32(bf16* dst, const float* v, int valid_cols) {
  if (valid_cols >= 32 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 pk;
      uint32_t* w = reinterpret_cast<uint32_t*>(&pk);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(v[q * 8 + 2 * i], v[q * 8 + 2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&b2);
      }
      reinterpret_cast<uint4*>(dst)[q] = pk;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < valid_cols) dst[i] = __float2bfloat16_rn(v[i]);
  }
}

// Warp-cooperative store of 32 16-bit values per lane: lane l's row is
// dst0 + l * ld (the warp's rows; rows >= nrows and columns >= nv are not
// written).  Every lane of the warp calls it (warp-uniform arguments except v).
// xs: the warp's slot; the 16-byte piece q of row r sits at r * 64 + 16 (q ^
// ((r >> 1) & 3)), so 8 consecutive lanes hit 8 different bank groups both
// when a lane writes its row and when 4 lanes read one row.
template <typename T>
__device__ __forceinline__ void store16_warp(uint8_t* xs, T* dst0, long long ld, const float* v, int nv,
                                             int nrows, int lane) {
  static_assert(sizeof(T) == 2, "16-bit output");
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 pk;
    uint32_t* w = reinterpret_cast<uint32_t*>(&pk);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if constexpr (std::is_same<T, bf16>::value) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(v[q * 8 + 2 * i], v[q * 8 + 2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&b2);
      } else {
        __half2 h2 = __floats2half2_rn(v[q * 8 + 2 * i], v[q * 8 + 2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t*>(&h2);
      }
    }
    *reinterpret_cast<uint4*>(xs + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4)) = pk;
  }
  __syncwarp();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = 8 * k + (lane >> 2), q = lane & 3;
    const uint4 x = *reinterpret_cast<const uint4*>(xs + r * 64 + ((q ^ ((r >> 1) & 3)) << 4));
    if (r < nrows && 8 * q < nv) *reinterpret_cast<uint4*>(dst0 + (long long)r * ld + 8 * q) = x;
  }
  __syncwarp();
}

// h += v * rs on 32 columns (col % 4 == 0) of this thread's row of the
// row-blocked residual Hs (one slot); v receives the new residual values.
// Consecutive 4-column groups of a row are 128 floats apart.
__device__ __forceinline__ void resid_add32(float* Hs, int row, int col, int d, float* v, float rs, int valid_cols) {
  if (valid_cols >= 32) {
    float4* H4 = reinterpret_cast<float4*>(Hs + h_blocked_offset(row, col, d));
    float4 o[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) o[q] = H4[q * 32];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      o[q].x = fmaf(v[4 * q], rs, o[q].x);
      o[q].y = fmaf(v[4 * q + 1], rs, o[q].y);
      o[q].z = fmaf(v[4 * q + 2], rs, o[q].z);
      o[q].w = fmaf(v[4 * q + 3], rs, o[q].w);
      v[4 * q] = o[q].x; v[4 * q + 1] = o[q].y; v[4 * q + 2] = o[q].z; v[4 * q + 3] = o[q].w;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) H4[q * 32] = o[q];
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (i < valid_cols) {
        float* hp = Hs + h_blocked_offset(row, col + i, d);
        const float o = fmaf(v[i], rs, *hp);
        *hp = o;
        v[i] = o;
      }
    }
  }
}

// The 32 residual values of columns col .. col+31 (col % 4 == 0) of this
// thread's row in the row-blocked layout: 8 groups of 4, 128 floats apart.
__device__ __forceinline__ void load_h8(const float* Hs, int row, int col, int d, float4* dst) {
  const float4* H4 = reinterpret_cast<const float4*>(Hs + h_blocked_offset(row, col, d));
#pragma unroll
  for (int q = 0; q < 8; ++q) dst[q] = H4[q * 32];
}

// Epilogue of one accumulator tile for this thread's row.  Every tcgen05.ld
// is executed by the whole warp (warp-uniform loops); only the stores are
// guarded by the row/column bounds.
// 32 consecutive accumulator columns (col .. col+31) of this thread's row:
// from TMEM (warp-collective), or, for the transposed ragged tile, from the
// thread's row of the shared-memory staging area.
__device__ __forceinline__ void acc_ld32(uint32_t tbase, const float* srow, int col, float* v) {
  if (srow) {
    const float4* s4 = reinterpret_cast<const float4*>(srow + col);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 x = s4[q];
      v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
    }
  } else {
    tmem_ld32(tbase + (uint32_t)col, v);
  }
}

// RMSNorm row scale from the per-tile partial sums of squares.
__device__ __forceinline__ float norm_row_scale(const TcGemmParams& p, int slot, int row) {
  const float* part = p.rsq + (long long)slot * p.rsq_slot_stride + row;
  float ss = 0.f;
  for (int i = 0; i < p.rsq_parts; ++i) ss += part[(long long)i * p.rsq_pitch];
  return rsqrtf(ss / (float)p.norm_dim + p.norm_eps);
}

// hpre: residual epilogues only, the tile's first 32-column chunk of this
// thread's row, loaded by the caller before it waited for the accumulator
// (so that load's latency hides behind the main loop).  srow: null, or this
// row of the transposed ragged tile's staging area (then tbase is unused).
// xs: this warp's output slot, or null for direct 16-bit stores.
template <int BN, int EPI>
__device__ __forceinline__ void run_epilogue(const TcGemmParams& p, uint32_t tbase, const NodeEntry& nd, int row,
                                             bool valid, int nb, int half, const float4* hpre,
                                             const float* srow, uint8_t* xs) {
  const int slot = nd.z;
  const long long rofs = (long long)row;
  // the warp's rows: lanes own consecutive rows; rows >= M are not stored
  const int lane = threadIdx.x & 31;
  const int wrow0 = row - lane;
  const int nrows = min(32, p.M - wrow0);
  // slot stores write 8-column pieces: 16-byte aligned rows and a column count
  // that is a multiple of 8 (warp-uniform decision)
  const int out_cols = EPI == TC_EPI_SWIGLU ? p.f_out : p.N;
  const bool via_slot = xs != nullptr && (p.ldc & 7) == 0 && (out_cols & 7) == 0 &&
                        (reinterpret_cast<uintptr_t>(p.C) & 15) == 0;
  if constexpr (EPI == TC_EPI_F32) {
    float rs = 1.f;
    if (p.rsq && valid) rs = norm_row_scale(p, slot, p.rsq_row0 + row);
#pragma unroll 1
    for (int c = half * (BN / 64); c < (half + 1) * (BN / 64); ++c) {
      float v[32];
      acc_ld32(tbase, srow, c * 32, v);
      const int col = nb * BN + c * 32;
      if (!valid || col >= p.N) continue;
      float* C = reinterpret_cast<float*>(p.C) + (long long)slot * p.c_slot_stride + rofs * p.ldc + col;
      if (p.rsq) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= rs;
      }
      store_f32x32(C, v, p.N - col);
    }
  } else if constexpr (EPI == TC_EPI_RESID || EPI == TC_EPI_RESID_ACT) {
    // h += acc * rs.  The residual of the next 32-column chunk is loaded while
    // the current one is processed (the epilogue is bound by that load's
    // latency, not by bandwidth).
    float rs = 1.f;
    if (p.rowscale && valid) rs = p.rowscale[(long long)slot * p.rs_slot_stride + row];
    const bool to_out = EPI == TC_EPI_RESID_ACT && p.out && nd.y == p.out_layer && row < p.seg_len;
    float* Hs = p.h + (long long)slot * p.h_slot_stride;
    constexpr int NCH = BN / 64;   // chunks per half tile
    const int c0 = half * NCH;
    auto full_chunk = [&](int c) { return valid && nb * BN + (c + 1) * 32 <= p.N; };
    float4 hn[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) hn[q] = hpre[q];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
      const int c = c0 + k;
      float4 hc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) hc[q] = hn[q];
      if (k + 1 < NCH && full_chunk(c + 1)) load_h8(Hs, row, nb * BN + (c + 1) * 32, p.ldh, hn);
      float v[32];
      acc_ld32(tbase, srow, c * 32, v);
      const int col = nb * BN + c * 32;
      if (col >= p.N) continue;   // warp-uniform; rows past M skip the residual below
      const int nv = p.N - col;
      if (valid) {
        if (nv >= 32) {
          float4* H4 = reinterpret_cast<float4*>(Hs + h_blocked_offset(row, col, p.ldh));
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float4 o = hc[q];
            o.x = fmaf(v[4 * q], rs, o.x);
            o.y = fmaf(v[4 * q + 1], rs, o.y);
            o.z = fmaf(v[4 * q + 2], rs, o.z);
            o.w = fmaf(v[4 * q + 3], rs, o.w);
            H4[q * 32] = o;
            v[4 * q] = o.x; v[4 * q + 1] = o.y; v[4 * q + 2] = o.z; v[4 * q + 3] = o.w;
          }
        } else {
          resid_add32(Hs, row, col, p.ldh, v, rs, nv);
        }
        if (p.rsq) {
#pragma unroll
          for (int i = 0; i < 32; ++i) ss = (i < nv) ? fmaf(v[i], v[i], ss) : ss;
        }
      }
      if (EPI == TC_EPI_RESID_ACT) {
        f16* X = reinterpret_cast<f16*>(p.C) + (long long)slot * p.c_slot_stride + rofs * p.ldc + col;
        if (via_slot)
          store16_warp(xs, X - (long long)lane * p.ldc, p.ldc, v, nv, nrows, lane);
        else if (valid)
          store_act32(X, v, nv);
        if (to_out) {
          bf16* O = reinterpret_cast<bf16*>(p.out) + ((long long)nd.x * p.seg_len + row) * p.N + col;
          store_bf16_32(O, v, nv);
        }
      }
    }
    if (p.rsq && valid)
      p.rsq[(long long)slot * p.rsq_slot_stride + (long long)(2 * nb + half) * p.rsq_pitch + row] = ss;
  } else if constexpr (EPI == TC_EPI_QKV_ROPE) {
    // heads of head_dim columns; pairs (j, j + hd/2) live in chunks (c1, c1 + hd/64)
    const int hd = p.head_dim;
    const int cph = hd / 32;          // chunks per head
    const int pairs = hd / 64;        // chunk pairs per head
    const float rs = (p.rsq && valid) ? norm_row_scale(p, slot, row) : 1.f;
    const int heads_half = BN / hd / 2;
#pragma unroll 1
    for (int hh = half * heads_half; hh < (half + 1) * heads_half; ++hh) {
      const int head = (nb * BN) / hd + hh;
      const bool rot = head < p.rope_heads;
#pragma unroll 1
      for (int pc = 0; pc < pairs; ++pc) {
        const int c1 = hh * cph + pc, c2 = c1 + pairs;
        float v1[32], v2[32];
        acc_ld32(tbase, srow, c1 * 32, v1);
        acc_ld32(tbase, srow, c2 * 32, v2);
        const int col1 = nb * BN + c1 * 32, col2 = nb * BN + c2 * 32;
        if (col1 >= p.N) continue;   // warp-uniform; rows past M are computed but not stored
        if (rot) {
          // frequency-major table: the warp's 32 rows read 32 consecutive entries
          // (rows past M read row 0's)
          const float2* cs = p.rope + (long long)(pc * 32) * p.rope_pitch + (valid ? row : 0);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float2 a = cs[(long long)i * p.rope_pitch];
            const float x1 = v1[i] * rs, x2 = v2[i] * rs;
            v1[i] = x1 * a.x - x2 * a.y;
            v2[i] = x2 * a.x + x1 * a.y;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            v1[i] *= rs;
            v2[i] *= rs;
          }
        }
        // value heads go only to V^T when it is requested (its reader takes V^T)
        if (!(p.vt && !rot)) {
          f16* C = reinterpret_cast<f16*>(p.C) + (long long)slot * p.c_slot_stride + rofs * p.ldc;
          if (via_slot) {
            f16* C0 = C - (long long)lane * p.ldc;
            store16_warp(xs, C0 + col1, p.ldc, v1, p.N - col1, nrows, lane);
            if (col2 < p.N) store16_warp(xs, C0 + col2, p.ldc, v2, p.N - col2, nrows, lane);
          } else if (valid) {
            store_act32(C + col1, v1, p.N - col1);
            if (col2 < p.N) store_act32(C + col2, v2, p.N - col2);
          }
        }
        if (p.vt && !rot && valid) {
          // value head: dims pc*32.. and hd/2 + pc*32.. of this row, transposed
          const int vh = head - p.rope_heads;
          f16* vt = p.vt + (((long long)slot * p.n_vheads + vh) * hd) * p.vt_pitch + row;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            vt[(long long)(pc * 32 + i) * p.vt_pitch] = __float2half_rn(v1[i]);
            vt[(long long)(hd / 2 + pc * 32 + i) * p.vt_pitch] = __float2half_rn(v2[i]);
          }
        }
      }
    }
  } else if constexpr (EPI == TC_EPI_SWIGLU) {
    // tile columns [0, BN/2) = gate features f0.., [BN/2, BN) = up features f0..
    constexpr int HALF = BN / 2;
    const int f0 = nb * HALF;
    const float rs = (p.rsq && valid) ? norm_row_scale(p, slot, row) : 1.f;
#pragma unroll 1
    for (int c = half * (HALF / 64); c < (half + 1) * (HALF / 64); ++c) {
      float g[32], u[32];
      acc_ld32(tbase, srow, c * 32, g);
      acc_ld32(tbase, srow, HALF + c * 32, u);
      const int f = f0 + c * 32;
      if (f >= p.f_out) continue;   // warp-uniform; rows past M are computed but not stored
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float gi = g[i] * rs;
        g[i] = gi / (1.f + __expf(-gi)) * (u[i] * rs);
      }
      f16* C = reinterpret_cast<f16*>(p.C) + (long long)slot * p.c_slot_stride + rofs * p.ldc + f;
      if (via_slot)
        store16_warp(xs, C - (long long)lane * p.ldc, p.ldc, g, p.f_out - f, nrows, lane);
      else if (valid)
        store_act32(C, g, p.f_out - f);
    }
  }
}

template <int BN, int EPI, bool TF32 = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmAs, const TcGemmParams p) {
  // tmAs: A with a SWAP_ROWS-row box (transposed ragged tile; unused otherwise)
  constexpr int BKE = TF32 ? BK / 2 : BK;   // elements per 128-byte k-block
  using SM = Smem<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::BAR_OFFSET);
  uint64_t* empty = full + SM::STAGES;
  uint64_t* tfull = empty + SM::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* stg_full = drain + 1;    // transposed ragged tile: D^T staged (all epilogue threads arrive)
  uint64_t* stg_empty = drain + 2;   // ... and read (the 64 threads of TMEM quarter 0 arrive)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  grid_dependency_sync();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // an earlier kernel of this forward already gave up on a wait: do nothing
  // (the forward's result is reported as failed), so a systematic failure
  // costs one bounded wait, not one per CTA and launch
  // (one thread reads the word, so the whole CTA takes the same decision)
  __shared__ unsigned skip_cta;
  if (threadIdx.x == 0) skip_cta = *reinterpret_cast<volatile unsigned*>(p.err) & ERR_WAIT_TIMEOUT_MASK;
  __syncthreads();
  if (skip_cta) return;
  if (threadIdx.x == 0) {
    for (int s = 0; s < SM::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], EPI_WARPS);
    }
    mbar_init(drain, 1);
    mbar_init(stg_full, 32 * EPI_WARPS);
    mbar_init(stg_empty, 64);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(2 * BN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int tiles_per_node = p.m_tiles * p.n_tiles;
  const int total = p.n_nodes * tiles_per_node;

  if (warp == 0) {
    {
      // ---------------- TMA producer (whole warp; one elected lane issues) ----------------
      const bool issuer = elect_one();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0;   // bit s: stage s has an issued load not yet seen complete by the consumer
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const int node = t / tiles_per_node, r = t - node * tiles_per_node;
        const int nb = r / p.m_tiles, mb = r - nb * p.m_tiles;
        const NodeEntry nd = p.nodes[node];
        const int a_outer = p.a_by_layer ? nd.y : nd.z;
        const bool swapped = SM::SWAP && p.swap_tail && mb == p.m_tiles - 1;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait_warp(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
          armed &= ~(1u << stage);
          uint8_t* sa = smem + stage * SM::STAGE_BYTES;
          if (!p.debug_no_loads) {
            if (issuer) mbar_expect_tx(&full[stage], swapped ? SM::SWAP_A_BYTES + SM::B_BYTES : SM::STAGE_BYTES);
            if (issuer)
              tma_load_3d(swapped ? &tmAs : &tmA, &full[stage], sa, kb * BKE, p.row0 + mb * BM, a_outer);
            if (issuer) tma_load_3d(&tmB, &full[stage], sa + SM::A_BYTES, kb * BKE, nb * BN, nd.y);
            armed |= 1u << stage;
          }
          if (++stage == SM::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        if (issuer) atomicOr(p.err, 1u);
        *abort_flag = 1;
      }
      // drain: wait (bounded) until every issued copy has landed
      if (*abort_flag) {
        for (int s = 0; s < SM::STAGES; ++s) {
          if (!(armed & (1u << s))) continue;
          const unsigned long long t0 = global_ns();
          // the latest phase of stage s is either complete or will complete; poll both parities
          while (!mbar_try_wait(&full[s], 0) && !mbar_try_wait(&full[s], 1)) {
            if (global_ns() - t0 > WAIT_LIMIT_NS) break;
          }
        }
      }
    }
  } else if (warp == 1) {
    {
      // ---------------- MMA issuer (whole warp; one elected lane issues) ----------------
      const bool issuer = elect_one();
      const uint32_t IDESC = TF32 ? idesc_tf32(BN) : idesc_f16(BN, p.ab_bf16);
      // transposed ragged tile: M = 128 weight rows, N = SWAP_ROWS activation rows
      const uint32_t IDESC_SW = TF32 ? idesc_tf32(SWAP_ROWS) : idesc_f16(SWAP_ROWS, p.ab_bf16);
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const int mb = (t % tiles_per_node) % p.m_tiles;
        const bool swapped = SM::SWAP && p.swap_tail && mb == p.m_tiles - 1;
        if (!mbar_wait_warp(&tempty[buf], acc_phase ^ 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait_warp(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * SM::STAGE_BYTES);
          const uint32_t sb = sa + SM::A_BYTES;
          if (swapped) {
            // D^T[128 j + f][r] (TMEM columns j SWAP_ROWS + r) = B rows 128 j + f times A rows r
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
#pragma unroll
              for (int j = 0; j < BN / 128; ++j) {
                const uint32_t dj = d_tmem + (uint32_t)(j * SWAP_ROWS);
                const uint64_t wdesc = sw128_desc(sb + j * 128 * 128 + kk * 32);
                const uint64_t xdesc = sw128_desc(sa + kk * 32);
                if constexpr (TF32) {
                  if (issuer) mma_tf32(dj, wdesc, xdesc, IDESC_SW, (kb > 0 || kk > 0) ? 1u : 0u);
                } else {
                  if (issuer) mma_f16(dj, wdesc, xdesc, IDESC_SW, (kb > 0 || kk > 0) ? 1u : 0u);
                }
              }
            }
          } else {
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {   // 32 bytes of the k-block per instruction
            if constexpr (TF32) {
              if (issuer) mma_tf32(d_tmem, sw128_desc(sa + kk * 32), sw128_desc(sb + kk * 32), IDESC,
                                   (kb > 0 || kk > 0) ? 1u : 0u);
            } else {
              if (issuer) mma_f16(d_tmem, sw128_desc(sa + kk * 32), sw128_desc(sb + kk * 32), IDESC,
                                  (kb > 0 || kk > 0) ? 1u : 0u);
            }
          }
          }
          if (issuer) mma_commit(&empty[stage]);
          if (++stage == SM::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (issuer) mma_commit(&tfull[buf]);
        if (++buf == 2) { buf = 0; acc_phase ^= 1; }
      }
      if (!ok) {
        if (issuer) atomicOr(p.err, 2u);
        *abort_flag = 1;
      }
      // make sure no MMA is still writing TMEM before it is freed
      if (issuer) mma_commit(drain);
      const unsigned long long t0 = global_ns();
      while (!mbar_try_wait(drain, 0)) {
        if (global_ns() - t0 > WAIT_LIMIT_NS) break;
      }
    }
  } else {
    // ---------------- epilogue (warps 2..9) ----------------
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
    const int half = (warp - 2) >> 2;        // which half of the tile's columns
    const int row_in_tile = quarter * 32 + lane;
    uint8_t* xs = smem + SM::XS_OFFSET + (warp - 2) * XS_SLOT;   // this warp's 16-bit output slot
    int buf = 0;
    uint32_t acc_phase = 0;
    uint32_t stg_phase = 0;   // transposed ragged tiles seen so far, mod 2
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      const int node = t / tiles_per_node, r = t - node * tiles_per_node;
      const int nb = r / p.m_tiles, mb = r - nb * p.m_tiles;
      const bool swapped = SM::SWAP && p.swap_tail && mb == p.m_tiles - 1;
      const NodeEntry nd = p.nodes[node];
      const int row = p.row0 + mb * BM + row_in_tile;
      const bool valid = row < p.M;
      float4 hpre[8];   // residual epilogues: first chunk of the row, loaded ahead of the wait
      if constexpr (EPI == TC_EPI_RESID || EPI == TC_EPI_RESID_ACT) {
        const int col = nb * BN + half * (BN / 2);
        if (valid && col + 32 <= p.N)
          load_h8(p.h + (long long)nd.z * p.h_slot_stride, row, col, p.ldh, hpre);
      }
      const bool got = mbar_wait(&tfull[buf], acc_phase, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) atomicOr(p.err, 4u);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
      if (swapped) {
        if constexpr (SM::SWAP) {
          // D^T: this warp's TMEM lanes are weight rows 128 half + 32 quarter + lane of the
          // tile, its columns half * SWAP_ROWS .. the activation rows; staged as
          // stg[row][column] once the previous transposed tile's rows have been read
          float* stg = reinterpret_cast<float*>(smem + SM::STG_OFFSET);
          if (!__all_sync(0xffffffffu, mbar_wait(stg_empty, stg_phase ^ 1, abort_flag))) {
            if (lane == 0) atomicOr(p.err, 4u);
            *abort_flag = 1;
            break;
          }
          if (half < BN / 128) {
            float v[SWAP_ROWS];
            tmem_ld16(tbase + (uint32_t)(half * SWAP_ROWS), v);
            const int col = half * 128 + quarter * 32 + lane;
#pragma unroll
            for (int i = 0; i < SWAP_ROWS; ++i) stg[i * SM::STG_PITCH + col] = v[i];
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);   // TMEM buffer free for the next tile
          mbar_arrive(stg_full);
          if (quarter == 0) {
            if (!__all_sync(0xffffffffu, mbar_wait(stg_full, stg_phase, abort_flag))) {
              if (lane == 0) atomicOr(p.err, 4u);
              *abort_flag = 1;
              break;
            }
            // lanes >= SWAP_ROWS own rows past M (nothing is stored for them): they
            // read staged row 0, so every read stays inside the SWAP_ROWS-row area
            const float* srow = stg + (lane < SWAP_ROWS ? lane : 0) * SM::STG_PITCH;
            run_epilogue<BN, EPI>(p, 0u, nd, row, valid, nb, half, hpre, srow, xs);
            mbar_arrive(stg_empty);
          }
          stg_phase ^= 1;
        }
      } else {
        run_epilogue<BN, EPI>(p, tbase, nd, row, valid, nb, half, hpre, nullptr, xs);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
      }
      if (++buf == 2) { buf = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(2 * BN) : "memory");
  }
}

// ---------------------------------------------------------------------------
// CTA-pair variant (cluster of 2, tcgen05 cta_group::2) for 256-column tiles:
// a pair computes 256 rows x 256 columns.  Each CTA loads its own 128 rows of
// A and its half (128 rows) of the B tile, so per CTA a pipeline stage is
// 32 KB instead of 48 KB and every B byte is fetched once per 256 output
// rows: less shared-memory and L2 traffic per multiply-add than one CTA per
// 128 x 256 tile.  The even CTA's single MMA thread issues
// tcgen05.mma.cta_group::2 (M = 256); each CTA's accumulator rows land in its
// own TMEM, so the epilogue is the one-CTA epilogue unchanged.
//   full[s]   (even CTA) both CTAs' copies of stage s, counted in bytes
//   empty[s]  (each CTA) stage s consumed (multicast commit)
//   tfull[b]  (each CTA) accumulator b complete (multicast commit)
//   tempty[b] (even CTA) accumulator b drained by both CTAs' epilogues
// Rows [row0, row0 + 256 m_tiles) of every node; the caller covers a ragged
// rest with the one-CTA kernel.  Every wait is bounded; the only unbounded
// waits are the two cluster barriers that every thread reaches.
struct SmemPair {
  static constexpr int A_BYTES = BM * BK * 2;        // this CTA's 128 rows
  static constexpr int B_BYTES = 128 * BK * 2;       // this CTA's 128 of the tile's 256 B rows
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = 6;
  static constexpr int BAR_OFFSET = STAGES * STAGE_BYTES;
  static constexpr int TOTAL = BAR_OFFSET + 256 + 1024;
};

__device__ __forceinline__ uint32_t ld_shared_cluster_u32(uint32_t cluster_addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const TcGemmParams p) {
  using SM = SmemPair;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::BAR_OFFSET);
  uint64_t* empty = full + SM::STAGES;
  uint64_t* tfull = empty + SM::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* skip_word = tmem_slot + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < SM::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    // an earlier kernel of this forward already gave up on a wait: the pair
    // skips its work (the even CTA decides for both)
    *skip_word = *reinterpret_cast<volatile unsigned*>(p.err) & ERR_WAIT_TIMEOUT_MASK;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();   // both CTAs' barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const bool skip = ld_shared_cluster_u32(mapa_shared(smem_u32(skip_word), 0)) != 0;

  const int tiles_per_node = p.m_tiles * p.n_tiles;
  const int total = p.n_nodes * tiles_per_node;
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;

  if (skip) {
    // nothing to do
  } else if (warp == 0) {
    {
      // ---------------- TMA producer (both CTAs; whole warp, one elected lane issues) ----------------
      const bool issuer = elect_one();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0;
      bool ok = true;
      const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);   // the even CTA's full[0]
      for (int t = cid; t < total && ok; t += ncl) {
        const int node = t / tiles_per_node, r = t - node * tiles_per_node;
        const int nb = r / p.m_tiles, mp = r - nb * p.m_tiles;
        const NodeEntry nd = p.nodes[node];
        const int a_outer = p.a_by_layer ? nd.y : nd.z;
        const int arow = p.row0 + mp * 256 + (int)rank * BM;
        const int brow = nb * 256 + (int)rank * 128;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait_cluster_warp(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
          armed &= ~(1u << stage);
          uint8_t* sa = smem + stage * SM::STAGE_BYTES;
          if (leader && issuer) mbar_expect_tx(&full[stage], 2 * SM::STAGE_BYTES);   // both CTAs' copies
          const uint32_t fb = full0 + (uint32_t)(stage * sizeof(uint64_t));
          if (issuer) tma_load_3d_pair(&tmA, fb, sa, kb * BK, arow, a_outer);
          if (issuer) tma_load_3d_pair(&tmB, fb, sa + SM::A_BYTES, kb * BK, brow, nd.y);
          armed |= 1u << stage;
          if (++stage == SM::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        if (issuer) atomicOr(p.err, 1u);
        *abort_flag = 1;
      }
      if (*abort_flag && leader) {   // copies of both CTAs are counted on the even CTA's barriers
        for (int s = 0; s < SM::STAGES; ++s) {
          if (!(armed & (1u << s))) continue;
          const unsigned long long t0 = global_ns();
          while (!mbar_try_wait_cluster(&full[s], 0) && !mbar_try_wait_cluster(&full[s], 1)) {
            if (global_ns() - t0 > WAIT_LIMIT_NS) break;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (leader) {
      // ---------------- MMA issuer (even CTA; whole warp, one elected lane issues) ----------------
      const bool issuer = elect_one();
      const uint32_t IDESC = idesc_f16(256, p.ab_bf16, 256);
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = cid; t < total && ok; t += ncl) {
        if (!mbar_wait_cluster_warp(&tempty[buf], acc_phase ^ 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * 256);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait_cluster_warp(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * SM::STAGE_BYTES);
          const uint32_t sb = sa + SM::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            if (issuer) mma_f16_pair(d_tmem, sw128_desc(sa + kk * 32), sw128_desc(sb + kk * 32), IDESC,
                         (kb > 0 || kk > 0) ? 1u : 0u);
          if (issuer) mma_commit_pair(&empty[stage], 0x3);
          if (++stage == SM::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (issuer) mma_commit_pair(&tfull[buf], 0x3);
        if (++buf == 2) { buf = 0; acc_phase ^= 1; }
      }
      if (!ok) {
        if (issuer) atomicOr(p.err, 2u);
        *abort_flag = 1;
      }
      if (issuer) mma_commit_pair(drain, 0x1);   // no MMA writes either CTA's TMEM after this arrives
      const unsigned long long t0 = global_ns();
      while (!mbar_try_wait(drain, 0)) {
        if (global_ns() - t0 > WAIT_LIMIT_NS) break;
      }
    }
  } else {
    // ---------------- epilogue (warps 2..9, both CTAs) ----------------
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
    int buf = 0;
    uint32_t acc_phase = 0;
    for (int t = cid; t < total; t += ncl) {
      const int node = t / tiles_per_node, r = t - node * tiles_per_node;
      const int nb = r / p.m_tiles, mp = r - nb * p.m_tiles;
      const NodeEntry nd = p.nodes[node];
      const int row = p.row0 + mp * 256 + (int)rank * BM + row_in_tile;
      const bool valid = row < p.M;
      float4 hpre[8];
      if constexpr (EPI == TC_EPI_RESID || EPI == TC_EPI_RESID_ACT) {
        const int col = nb * 256 + half * 128;
        if (valid && col + 32 <= p.N)
          load_h8(p.h + (long long)nd.z * p.h_slot_stride, row, col, p.ldh, hpre);
      }
      const bool got = mbar_wait_cluster(&tfull[buf], acc_phase, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) atomicOr(p.err, 4u);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * 256);
      run_epilogue<256, EPI>(p, tbase, nd, row, valid, nb, half, hpre, nullptr, nullptr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0 + (uint32_t)(buf * sizeof(uint64_t)));
      if (++buf == 2) { buf = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  cluster_sync_all();   // no MMA, copy or epilogue of either CTA still uses TMEM or shared memory
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512) : "memory");
  }
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 get_tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

namespace {

template <int BN, int EPI, bool TF32 = false>
cudaError_t launch_kernel(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tas,
                          const TcGemmParams& p, int sm_count, cudaStream_t st) {
  using SM = Smem<BN>;
  const int total = p.n_nodes * p.m_tiles * p.n_tiles;
  const int grid = total < sm_count ? total : sm_count;
  return launch_pdl(tc_gemm_kernel<BN, EPI, TF32>, dim3(grid), dim3(NUM_THREADS), SM::TOTAL, st, ta, tb, tas, p);
}

template <int BN, int EPI, bool TF32 = false>
cudaError_t configure() {
  return cudaFuncSetAttribute(tc_gemm_kernel<BN, EPI, TF32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              Smem<BN>::TOTAL);
}

// Clusters of the pair kernel that fit on the device at once (persistent grid).
template <int EPI>
int& pair_clusters() {
  static int n = 0;
  return n;
}

template <int EPI>
cudaError_t configure_pair() {
  cudaError_t e = cudaFuncSetAttribute(tc_gemm_pair_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SmemPair::TOTAL);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = SmemPair::TOTAL;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2; attr.val.clusterDim.y = 1; attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  // a device or driver that cannot place the pairs leaves them unused (the
  // one-CTA kernel covers every row then)
  if (cudaOccupancyMaxActiveClusters(&n, tc_gemm_pair_kernel<EPI>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  pair_clusters<EPI>() = n;
  return cudaSuccess;
}

bool pair_available(int epi) {
  switch (epi) {
    case TC_EPI_F32: return pair_clusters<TC_EPI_F32>() > 0;
    case TC_EPI_RESID: return pair_clusters<TC_EPI_RESID>() > 0;
    case TC_EPI_RESID_ACT: return pair_clusters<TC_EPI_RESID_ACT>() > 0;
    case TC_EPI_QKV_ROPE: return pair_clusters<TC_EPI_QKV_ROPE>() > 0;
    case TC_EPI_SWIGLU: return pair_clusters<TC_EPI_SWIGLU>() > 0;
    default: return false;
  }
}

template <int EPI>
cudaError_t launch_pair(const CUtensorMap& ta, const CUtensorMap& tb, const TcGemmParams& p, cudaStream_t st) {
  const int total = p.n_nodes * p.m_tiles * p.n_tiles;
  const int cl = pair_clusters<EPI>();
  if (cl <= 0) return cudaErrorInvalidConfiguration;
  const int clusters = total < cl ? total : cl;
  tc_gemm_pair_kernel<EPI><<<2 * clusters, NUM_THREADS, SmemPair::TOTAL, st>>>(ta, tb, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t setup_tc_gemm() {
  static bool done = false;
  if (done) return cudaSuccess;
  if (!get_tensor_map_encoder()) return cudaErrorNotSupported;
  cudaError_t e = configure<256, TC_EPI_F32>();
  if (e == cudaSuccess) e = configure<128, TC_EPI_F32>();
  if (e == cudaSuccess) e = configure<64, TC_EPI_F32>();
  if (e == cudaSuccess) e = configure<256, TC_EPI_RESID>();
  if (e == cudaSuccess) e = configure<256, TC_EPI_RESID_ACT>();
  if (e == cudaSuccess) e = configure<256, TC_EPI_QKV_ROPE>();
  if (e == cudaSuccess) e = configure<256, TC_EPI_SWIGLU>();
  if (e == cudaSuccess) e = configure<256, TC_EPI_RESID_ACT, true>();
  if (e == cudaSuccess) e = configure<256, TC_EPI_F32, true>();
  if (e == cudaSuccess) e = configure<128, TC_EPI_F32, true>();
  if (e == cudaSuccess) e = configure<64, TC_EPI_F32, true>();
  if (e == cudaSuccess) e = configure_pair<TC_EPI_F32>();
  if (e == cudaSuccess) e = configure_pair<TC_EPI_RESID>();
  if (e == cudaSuccess) e = configure_pair<TC_EPI_RESID_ACT>();
  if (e == cudaSuccess) e = configure_pair<TC_EPI_QKV_ROPE>();
  if (e == cudaSuccess) e = configure_pair<TC_EPI_SWIGLU>();
  if (e == cudaSuccess) done = true;
  return e;
}

// 3-D tensor map over an array [outer][rows][inner] of 16-bit (fp16 / bf16)
// or fp32 elements (inner contiguous; consecutive outer indices pitch_rows
// rows apart), box = box_inner x box_rows x 1, 128-byte swizzle, zero fill
// out of bounds.  ty: 0 = fp16, 1 = bf16, 2 = fp32.
cudaError_t make_tmap_3d(CUtensorMap* map, const void* base, int inner, int rows, int outer, int box_inner,
                         int box_rows, int pitch_rows, int ty) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  if (pitch_rows <= 0) pitch_rows = rows;
  const cuuint64_t esz = ty == 2 ? 4 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)outer};
  cuuint64_t strides[2] = {(cuuint64_t)inner * esz, (cuuint64_t)inner * pitch_rows * esz};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt = ty == 2 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                         : (ty == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  CUresult r = enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 256-column tiles of 256 or more rows run on CTA pairs only when the
// environment sets ARMT_GEMM_CTA_PAIRS=1: on the 1B workload the pairs plus
// the one-CTA launch for the ragged rows measured slower (311.5 vs 321.5 ms
// per forward on one box) than one CTA per 128 x 256 tile.
bool tc_gemm_pairs_enabled() {
  static const bool on = [] {
    const char* v = getenv("ARMT_GEMM_CTA_PAIRS");
    return v && v[0] == '1';
  }();
  return on;
}

// The transposed ragged row tile is on unless the environment sets
// ARMT_GEMM_SWAP_TAIL=0 (for A/B measurement).
bool tc_gemm_swap_enabled() {
  static const bool on = [] {
    const char* v = getenv("ARMT_GEMM_SWAP_TAIL");
    return !(v && v[0] == '0');
  }();
  return on;
}

bool tc_gemm_supported(int m, int n, int k) {
  (void)m;
  return k % 8 == 0 && n % 16 == 0 && get_tensor_map_encoder() != nullptr;
}

namespace {

// Decide whether the last row tile runs transposed and, if so, build the A
// map with a SWAP_ROWS-row box (otherwise tas is a copy of ta, never read).
cudaError_t setup_swap_tail(const TcGemmOperands& op, TcGemmParams& p, int bn, int box_inner, int ty,
                            const CUtensorMap& ta, CUtensorMap* tas) {
  const int last_rows = p.M - p.row0 - (p.m_tiles - 1) * BM;
  p.swap_tail = (bn % 128 == 0 && last_rows <= SWAP_ROWS && tc_gemm_swap_enabled()) ? 1 : 0;
  if (!p.swap_tail) {
    *tas = ta;
    return cudaSuccess;
  }
  return make_tmap_3d(tas, op.A, p.K, op.a_rows, op.a_outer, box_inner, SWAP_ROWS, op.a_pitch, ty);
}

// fp32 operands on kind::tf32: k-blocks of 32 words; one-CTA kernel only
cudaError_t launch_tc_gemm_tf32(const TcGemmOperands& op, TcGemmParams p, int epi, int bn, int sm_count,
                                cudaStream_t st) {
  constexpr int BKE = BK / 2;
  CUtensorMap ta, tb;
  cudaError_t e = make_tmap_3d(&ta, op.A, p.K, op.a_rows, op.a_outer, BKE, BM, op.a_pitch, 2);
  if (e == cudaSuccess) e = make_tmap_3d(&tb, op.B, p.K, op.b_rows, op.b_outer, BKE, bn, 0, 2);
  if (e != cudaSuccess) return e;
  p.k_blocks = (p.K + BKE - 1) / BKE;
  p.row0 = 0;
  p.m_tiles = (p.M + BM - 1) / BM;
  p.n_tiles = (p.N + bn - 1) / bn;
  CUtensorMap tas;
  e = setup_swap_tail(op, p, bn, BKE, 2, ta, &tas);
  if (e != cudaSuccess) return e;
  if (bn == 256 && epi == TC_EPI_RESID_ACT)
    return launch_kernel<256, TC_EPI_RESID_ACT, true>(ta, tb, tas, p, sm_count, st);
  if (bn == 256 && epi == TC_EPI_F32) return launch_kernel<256, TC_EPI_F32, true>(ta, tb, tas, p, sm_count, st);
  if (bn == 128 && epi == TC_EPI_F32) return launch_kernel<128, TC_EPI_F32, true>(ta, tb, tas, p, sm_count, st);
  if (bn == 64 && epi == TC_EPI_F32) return launch_kernel<64, TC_EPI_F32, true>(ta, tb, tas, p, sm_count, st);
  return cudaErrorInvalidValue;
}

}  // namespace

int tc_pick_bn(int n) { return n >= 256 ? 256 : (n >= 128 ? 128 : 64); }

cudaError_t launch_tc_gemm(const TcGemmOperands& op, TcGemmParams p, int epi, int bn, int sm_count,
                           cudaStream_t st) {
  if (p.ab_tf32) return launch_tc_gemm_tf32(op, p, epi, bn, sm_count, st);
  CUtensorMap ta, tb;
  cudaError_t e = make_tmap_3d(&ta, op.A, p.K, op.a_rows, op.a_outer, BK, BM, op.a_pitch, p.ab_bf16 != 0);
  if (e != cudaSuccess) return e;
  p.k_blocks = (p.K + BK - 1) / BK;
  p.row0 = 0;
  if (bn == 256 && p.M >= 256 && tc_gemm_pairs_enabled() && pair_available(epi)) {
    // rows [0, 256 floor(M / 256)) on CTA pairs, the rest on the one-CTA kernel
    CUtensorMap tbp;
    e = make_tmap_3d(&tbp, op.B, p.K, op.b_rows, op.b_outer, BK, 128, 0, p.ab_bf16 != 0);
    if (e != cudaSuccess) return e;
    TcGemmParams pp = p;
    pp.m_tiles = p.M / 256;
    pp.n_tiles = (p.N + 255) / 256;
#define ARMT_TC_PAIR(E) \
    if (epi == E) e = launch_pair<E>(ta, tbp, pp, st);
    e = cudaErrorInvalidValue;
    ARMT_TC_PAIR(TC_EPI_F32)
    ARMT_TC_PAIR(TC_EPI_RESID)
    ARMT_TC_PAIR(TC_EPI_RESID_ACT)
    ARMT_TC_PAIR(TC_EPI_QKV_ROPE)
    ARMT_TC_PAIR(TC_EPI_SWIGLU)
#undef ARMT_TC_PAIR
    if (e != cudaSuccess) return e;
    p.row0 = pp.m_tiles * 256;
    if (p.row0 >= p.M) return cudaSuccess;
  }
  e = make_tmap_3d(&tb, op.B, p.K, op.b_rows, op.b_outer, BK, bn, 0, p.ab_bf16 != 0);
  if (e != cudaSuccess) return e;
  p.m_tiles = (p.M - p.row0 + BM - 1) / BM;
  p.n_tiles = (p.N + bn - 1) / bn;
  CUtensorMap tas;
  e = setup_swap_tail(op, p, bn, BK, p.ab_bf16 != 0, ta, &tas);
  if (e != cudaSuccess) return e;
#define ARMT_TC_CASE(BNV, E) \
  if (bn == BNV && epi == E) return launch_kernel<BNV, E>(ta, tb, tas, p, sm_count, st);
  ARMT_TC_CASE(256, TC_EPI_F32)
  ARMT_TC_CASE(128, TC_EPI_F32)
  ARMT_TC_CASE(64, TC_EPI_F32)
  ARMT_TC_CASE(256, TC_EPI_RESID)
  ARMT_TC_CASE(256, TC_EPI_RESID_ACT)
  ARMT_TC_CASE(256, TC_EPI_QKV_ROPE)
  ARMT_TC_CASE(256, TC_EPI_SWIGLU)
#undef ARMT_TC_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_tc_gemm_unit(int G, int m, int n, int k, const void* A, const void* B, int num_b,
                                const NodeEntry* nodes, float* C, unsigned* err, int ab, cudaStream_t st,
                                int debug_no_loads) {
  int dev = 0, sms = 148;
  cudaError_t se = setup_tc_gemm();
  if (se != cudaSuccess) return se;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  TcGemmOperands op;
  op.A = A; op.a_rows = m; op.a_outer = G;
  op.B = B; op.b_rows = n; op.b_outer = num_b;
  TcGemmParams p{};
  p.nodes = nodes; p.n_nodes = G; p.M = m; p.N = n; p.K = k;
  p.C = C; p.c_slot_stride = (long long)m * n; p.ldc = n;
  p.err = err;
  p.ab_bf16 = ab == 1;
  p.ab_tf32 = ab == 2;
  p.debug_no_loads = debug_no_loads;
  const int bn = tc_pick_bn(n);
  return launch_tc_gemm(op, p, TC_EPI_F32, bn, sms, st);
}

}  // namespace armt
