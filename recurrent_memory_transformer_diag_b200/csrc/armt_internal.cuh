// Internal declarations shared by the library's translation units.
// Nothing here is part of the C ABI (include/armt.h is).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <string>
#include <utility>
#include <vector>

#include "../../include/armt.h"

namespace armt {

typedef __nv_bfloat16 bf16;
typedef __half f16;

// Bits of the device error word (Workspace::err).
constexpr unsigned ERR_WAIT_TIMEOUT_MASK = 0x77u; // bits 0-2 (GEMM), 4-6 (attention): a bounded wait ran out

// Residual stream layout on the tensor-core path ("row-blocked"): rows in
// blocks of 32, each block stored as [d/4 column groups][32 rows][4 columns].
// Epilogue threads own one accumulator row each (32 consecutive rows per
// warp), so a 16-byte access of 4 columns by the 32 threads of a warp covers
// one contiguous 512-byte span instead of 32 separate rows.  d % 4 == 0;
// a slot holds rows_blocked(T') rows.
__host__ __device__ inline long long h_blocked_offset(int row, int col, int d) {
  return ((long long)(row >> 5) * (d >> 2) + (col >> 2)) * 128 + (row & 31) * 4 + (col & 3);
}
__host__ __device__ inline int rows_blocked(int Tp) { return (Tp + 31) & ~31; }

// Programmatic dependent launch.  The forward's kernels are launched with
// programmatic stream serialisation, so a kernel's blocks may be scheduled
// while its predecessor drains (hiding the launch gap); each such kernel
// starts with grid_dependency_sync(): it lets its own dependant be scheduled
// early, then waits until the predecessor grid has completed and its memory
// is visible, before touching any data.  Launched without the attribute, the
// wait returns at once.
__device__ __forceinline__ void grid_dependency_sync() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Whether the forward's kernels use programmatic dependent launch (only when
// the environment sets ARMT_PDL=1).
bool pdl_enabled();

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// One node of the (segment, layer) grid as the kernels see it: x = segment s,
// y = layer l, z = activation slot (s mod number-of-slots), w = flags.
typedef int4 NodeEntry;

// A contiguous run of node-table entries launched together (one wave).
struct Wave {
  int first;   // index of the wave's first entry in the device node table
  int count;   // nodes in the wave
  bool any_first_layer;
  int first_layer_pos;   // index within the wave of the (single) layer-0 node, -1 if none
  int first_layer_seg;   // its segment, -1 if none
  int last_layer_seg;    // segment of the wave's (single) last-layer node, -1 if none
  bool any_last_layer;
};

// Device workspace.  Activations are per slot: a segment keeps its slot for
// all its layers, and the <= L segments live in one wave have distinct slots.
struct Workspace {
  int slots = 0;
  int tp_max = 0;           // max rows per node (max_seg_len + n_mem)
  float* h = nullptr;       // residual stream, fp32: [slots][T'][d] (fp32 path), row-blocked
                            // [slots][rows_blocked(T')][d] (tensor-core path)
  void* xb = nullptr;       // [slots][T'][d] GEMM operand copy of h (fp32, or fp16 on the tensor-core path)
  float* qm = nullptr;      // [slots][T'][dk] memory-read query
  float* phi = nullptr;     // [slots][T'][P] DPFP features, fp32 (tf32-rounded on the tensor-core path)
  float* inv_den = nullptr; // [slots][T'] 1 / (z . phi + eps)
  float* rsq = nullptr;     // [slots][2 ceil(d/256)][T'] RMSNorm partial sums (tensor-core path)
  void* qkv = nullptr;      // [slots][T'][Nqkv]  (fp32 / fp16)
  void* attn = nullptr;     // [slots][T'][H*hd]  (fp32 / fp16)
  void* vt = nullptr;       // [slots][KV][hd][pitch] fp16 V^T for the tcgen05 attention
  void* gu = nullptr;       // [slots][T'][2F]    (fp32 path only)
  void* u = nullptr;        // [slots][T'][F]     (fp32 / fp16)
  float* kv = nullptr;      // [slots][M][kv_ld] = k | v | gate logit (gated write)
  float* phik = nullptr;    // [slots][M][P]
  float* gram = nullptr;    // [slots][M][M] phi_j . phi_j'
  float* coef = nullptr;    // [slots][M] 1 / (z_j . phi_j + eps)
  float* gamma = nullptr;   // [slots][M]
  float* beta = nullptr;    // [slots][M] write strength (gated write)
  float2* rope = nullptr;   // [hd/2][tp_max] (cos, sin), frequency-major
  NodeEntry* nodes = nullptr;
  int nodes_cap = 0;
  unsigned* err = nullptr;  // device error word (bounded waits)
};

// Device weights in the layout the grouped kernels read: fp32 on the fp32
// path; on the tensor-core path the bf16-rounded values stored as fp16 (fp16
// holds every bf16 value of magnitude >= 2^-17 exactly).
struct Weights {
  bool loaded = false;
  float* mem_emb = nullptr;  // [M][d] fp32
  void* w_qkv = nullptr;     // [L][Nqkv][d]   attn gain folded
  void* w_o = nullptr;       // [L][d][H*hd]
  void* w_gu = nullptr;      // [L][2F][d]     mlp gain folded; gate rows then up rows
  void* w_down = nullptr;    // [L][d][F]
  void* w_qm = nullptr;      // [L][dk][d]
  void* w_kvm = nullptr;     // [L][kv_ld][d]  key rows, value rows, gate row (gated write), zero rows
};

struct Dims {
  int L, d, H, KV, hd, F, M, dk, nu, P, nqkv;
  float theta, rms_eps, mem_eps;
  bool bf16;
  bool write_gate = false;   // beta_j = sigmoid(w_beta . m_j) scales each row's write of A
  bool clamp_gamma = true;   // gamma_j clamped to [0, 1]
};

// Columns of a projected memory row [k (dk) | v (d) | gate logit]: the gated
// write adds one column, padded to 16 so the projection keeps N % 16 == 0.
inline int kv_ld(const Dims& dm) { return dm.dk + dm.d + (dm.write_gate ? 16 : 0); }

}  // namespace armt

struct armt_ctx {
  armt_config cfg;
  armt::Dims dm;
  int device = 0;
  int sm_count = 0;
  bool use_graph = true;
  armt::Weights w;
  armt::Workspace ws;
  std::string last_error;
  // CUDA graph of the last forward
  cudaGraphExec_t graph_exec = nullptr;
  cudaStream_t capture_stream = nullptr;
  struct GraphKey {
    int S = -1, T = -1, sched = -1, carry = 0;
    const void* emb = nullptr; void* out = nullptr; float* A = nullptr; float* z = nullptr;
  } graph_key;
  // node table of the last (S, schedule)
  int table_S = -1, table_sched = -1;
  std::vector<armt::Wave> waves;
  // node table of the last layer-pipeline stage call (S, layer offset, total
  // layers); it shares the device table with the forward, so uploading one
  // invalidates the other
  int stage_S = -1, stage_offset = -1, stage_total = -1;
  std::vector<armt::Wave> stage_waves;
  // host-buffer forward staging
  void* st_emb = nullptr; void* st_out = nullptr; float* st_A = nullptr; float* st_z = nullptr;
  size_t st_tokens = 0;
  // host-buffer forward with page-locked buffers: one graph whose per-segment
  // input copies, waves and per-segment output copies run on three streams
  cudaGraphExec_t host_graph_exec = nullptr;
  GraphKey host_key;
  cudaStream_t copy_in_stream = nullptr, copy_out_stream = nullptr;
  std::vector<cudaEvent_t> host_events;
  // each wave's memory write on a second stream, overlapping the next wave's
  // first kernels (tensor-core path); ARMT_OVERLAP_WRITE=0 turns it off
  bool overlap_write = true;
  cudaStream_t ov_stream = nullptr;
  cudaEvent_t ov_ev[4] = {nullptr, nullptr, nullptr, nullptr};
};

namespace armt {

// ---- kernels launched by the scheduler (all take the wave's node pointer) ----

enum GemmEpi { EPI_STORE_F32 = 0, EPI_STORE_ACT = 1, EPI_RESID = 2 };

struct GemmArgs {
  const NodeEntry* nodes;
  int n_nodes;
  int M, N, K;
  const void* A; long long a_slot_stride; int lda; int a_by_layer;
  const void* B; long long b_layer_stride; int ldb;
  void* C; long long c_slot_stride; int ldc;
  const float* rowscale; long long rs_slot_stride;   // optional (nullptr)
  int epi;
};

// SIMT grouped GEMM, fp32 operands (fp32 path, unit entry points).
cudaError_t launch_simt_gemm(const GemmArgs& a, cudaStream_t st);

// fp32 path: h row-major.  Tensor-core path (xb != nullptr): h row-blocked,
// xb the fp16 copy, row-major.
cudaError_t launch_init_first_layer(const Dims& dm, const NodeEntry* nodes, int n, int T, int Tp,
                                    const void* emb, const float* mem_emb, float* h, f16* xb, cudaStream_t st);
// Tensor-core path: per-row sums of squares of the row-blocked residual into
// the RMSNorm partials rsq[slot][part][pitch] (part 0 the row's sum, the rest 0).
cudaError_t launch_row_sumsq(const Dims& dm, const NodeEntry* nodes, int n, int Tp, const float* h, float* rsq,
                             long long rsq_slot_stride, int parts, int pitch, cudaStream_t st);
// RMSNorm (no gain) of rows row0 .. row0+nrows-1 of every node's slot.
cudaError_t launch_rmsnorm(const Dims& dm, const NodeEntry* nodes, int n, int Tp, int row0, int nrows,
                           const float* h, void* xb, float eps, cudaStream_t st);
cudaError_t launch_dpfp_read(const Dims& dm, const NodeEntry* nodes, int n, int Tp, const float* qm,
                             const float* z_state, float* phi, float* inv_den, cudaStream_t st);
// rope: [hd/2][rope_pitch] (cos, sin) of angle p * theta^(-2j/hd) at [j][p]
cudaError_t launch_rope(const Dims& dm, const NodeEntry* nodes, int n, int Tp, void* qkv,
                        const float2* rope, int rope_pitch, cudaStream_t st);
cudaError_t launch_attention_simt(const Dims& dm, const NodeEntry* nodes, int n, int Tp,
                                  const void* qkv, void* out, cudaStream_t st);
cudaError_t launch_swiglu(const Dims& dm, const NodeEntry* nodes, int n, int Tp, const void* gu,
                          void* u, cudaStream_t st);
// shared memory of memw_phi (bytes)
size_t memw_phi_smem(const Dims& dm);
// kv rows of kv_ld(dm) columns; beta [slots][M] written (gated write) or unused
cudaError_t launch_memw_phi(const Dims& dm, const NodeEntry* nodes, int n, const float* kv,
                            float* z_state, float* phik, float* gram, float* coef, float* gamma, float* beta,
                            cudaStream_t st);
cudaError_t launch_memw_update(const Dims& dm, const NodeEntry* nodes, int n, const float* kv,
                               const float* phik, const float* gram, const float* coef, const float* beta,
                               float* A_state, cudaStream_t st);
// layer-pipeline hand-off rows of the node at local layer `layer` (see simt_kernels.cu)
cudaError_t launch_stage_rows_in(const Dims& dm, const NodeEntry* nodes, int n, int layer, int Tp, const float* in,
                                 float* h, void* xb, cudaStream_t st);
cudaError_t launch_stage_rows_out(const Dims& dm, const NodeEntry* nodes, int n, int layer, int Tp, const float* h,
                                  float* out, cudaStream_t st);
cudaError_t launch_output(const Dims& dm, const NodeEntry* nodes, int n, int T, int Tp,
                          const float* h, void* out, cudaStream_t st);

cudaError_t setup_memory_kernels(const Dims& dm);

// tcgen05 attention (head_dim 64 or 128): reads V^T [slot][KV][hd][vt_pitch]
bool attention_tc_supported(const Dims& dm);
int attention_tc_vt_pitch(int Tp);
cudaError_t setup_attention_tc();
cudaError_t launch_attention_tc(const Dims& dm, const NodeEntry* nodes, int n, int Tp, int slots, const void* qkv,
                                const void* vt, void* out, unsigned* err, cudaStream_t st);

// weight conversions at load: fp32 copy, or bf16 rounding (RNE) stored as fp16
// weight upload: fp32 copy; fp32 -> bf16 (RNE) held in fp16; fp32 -> fp16 (RNE)
enum ConvertMode { CONVERT_COPY_F32 = 0, CONVERT_BF16_AS_F16 = 1, CONVERT_F16 = 2 };
cudaError_t launch_convert(const float* src, void* dst, size_t n, int mode, cudaStream_t st);

}  // namespace armt
