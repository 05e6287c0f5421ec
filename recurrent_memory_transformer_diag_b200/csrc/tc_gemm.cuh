// Interface of the tcgen05 grouped GEMM (tc_gemm.cu).
#pragma once

#include "armt_internal.cuh"

namespace armt {

// Fused epilogues (thread = one accumulator row; see tc_gemm.cu).
enum TcEpi {
  TC_EPI_F32 = 0,        // C (fp32) = acc (times the RMSNorm row scale when rsq is set)
  TC_EPI_RESID = 1,      // h += acc * rowscale[row]   (rowscale optional)
  TC_EPI_RESID_ACT = 2,  // as RESID, and C (fp16) = new h (the next GEMM's operand); optional
                         // norm partials (rsq) and bf16 copy of rows < seg_len to `out`
  TC_EPI_QKV_ROPE = 3,   // C (fp16) = acc, rotate-half RoPE on heads < rope_heads
  TC_EPI_SWIGLU = 4      // C (fp16)[f] = silu(acc[gate f]) * acc[up f]; B rows interleaved per 128
};

struct TcGemmParams {
  const NodeEntry* nodes;
  int n_nodes;
  int M, N, K;              // per node: rows, B rows (output columns), reduction
  int m_tiles, n_tiles, k_blocks;
  int row0;                 // first row of the range this launch covers (rows row0 .. M-1)
  int a_by_layer;           // A's outer TMA coordinate: 0 = node slot, 1 = node layer
  int ab_bf16;              // 16-bit operand type: 0 = fp16, 1 = bf16 (both operands alike)
  int ab_tf32;              // 1: both operands fp32, multiplied at tf32 precision (kind::tf32)
  void* C; long long c_slot_stride; int ldc;
  float* h; long long h_slot_stride; int ldh;   // residual, row-blocked (h_blocked_offset), ldh = row length
  const float* rowscale; long long rs_slot_stride;
  const float2* rope; int rope_pitch; int rope_heads; int head_dim;   // rope [hd/2][rope_pitch]
  // QKV epilogue: write the value heads (heads >= rope_heads) transposed,
  // vt[slot][head - rope_heads][dim][row] with rows vt_pitch apart, instead of
  // into C (optional; without it they go to C like q and k)
  f16* vt; int vt_pitch; int n_vheads;
  int f_out;                // SWIGLU: number of valid output features
  // RMSNorm folded into the GEMMs.  Residual epilogues write, per row and per
  // half n-tile, the partial sum of squares of the new residual over those
  // columns (rsq[slot][2 * tile + half][row], parts rsq_pitch rows apart, so a
  // warp's 32 rows touch 32 consecutive floats); QKV,
  // gate/up and kv-mem epilogues scale their rows by
  // rsqrt(sum of the partials / norm_dim + eps).
  float* rsq; long long rsq_slot_stride; int rsq_parts; int rsq_pitch; int norm_dim; float norm_eps;
  int rsq_row0;             // F32 epilogue: output row r is normalised with the partials of row rsq_row0 + r
  // final hidden states (down-projection epilogue of last-layer nodes)
  void* out; int out_layer; int seg_len;
  unsigned* err;            // device error word (bounded waits)
  int swap_tail;            // 1: the last row tile (at most 16 rows) is computed transposed (set by the launcher)
  int debug_no_loads;       // test hook: the producer issues no copies, so the first wait for a stage
                            // cannot complete and the bounded-wait error path runs (never set by the forward)
};

struct TcGemmOperands {
  const void* A; int a_rows; int a_outer;   // [a_outer][a_rows][K] (rows a_pitch apart per outer step)
  const void* B; int b_rows; int b_outer;   // [b_outer][b_rows][K]; both 16-bit, or both fp32 (ab_tf32)
  int a_pitch = 0;                          // rows between outer steps of A (0 = a_rows)
};

cudaError_t setup_tc_gemm();
int tc_pick_bn(int n);
bool tc_gemm_pairs_enabled();
bool tc_gemm_swap_enabled();
bool tc_gemm_supported(int m, int n, int k);
cudaError_t launch_tc_gemm(const TcGemmOperands& op, TcGemmParams p, int epi, int bn, int sm_count,
                           cudaStream_t st);
// ab: 0 = fp16, 1 = bf16, 2 = fp32 operands on kind::tf32
cudaError_t launch_tc_gemm_unit(int G, int m, int n, int k, const void* A, const void* B, int num_b,
                                const NodeEntry* nodes, float* C, unsigned* err, int ab, cudaStream_t st,
                                int debug_no_loads = 0);

}  // namespace armt
