// C ABI of the Diagonal Batching ARMT forward: context, weight layout, the
// wave scheduler and CUDA-graph capture.
//
// Scheduler.  Node (s, l) depends only on (s, l-1) and (s-1, l), so wave
// i = s + l holds up to min(S, L) independent nodes (Pith review of arXiv
// 2506.05229, "What carries the argument"; Lemma 3.1: S + L - 1 waves is the
// minimum).  The host builds a node table once per (S, schedule) and uploads
// it; every kernel of a wave reads its node's (segment, layer, slot) from
// the table, picks that layer's weights from the stacked [L, ...] tensors
// and that segment's activations from its slot.  A segment keeps one slot
// (s mod min(S, L)) for all its layers, so a node updates its activations in
// place and no two nodes of a wave share a slot.  The sequential schedule
// uses the same kernels with one node per launch (the S x L baseline,
// Pith review Figure 3).  The whole forward is captured once in a CUDA graph
// and replayed (skill page "Practical Guidance": keep the per-layer memory
// state on the GPU and synchronise only at the end).
#include <cuda.h>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <cstdlib>
#include <vector>

#include "armt_internal.cuh"
#include "tc_gemm.cuh"

using namespace armt;

// Programmatic dependent launch is off unless ARMT_PDL=1: on the 1B forward it
// measured slower (334.3-335.3 ms against 325.5 ms without, same box).
bool armt::pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("ARMT_PDL");
    return v && v[0] == '1';
  }();
  return on;
}

namespace {

armt_status fail(armt_ctx* ctx, armt_status s, const char* what) {
  if (ctx) ctx->last_error = what;
  return s;
}

armt_status cuda_fail(armt_ctx* ctx, cudaError_t e, const char* where) {
  if (ctx) {
    ctx->last_error = std::string(where) + ": " + cudaGetErrorString(e);
  }
  cudaGetLastError();  // clear a sticky-free error so later calls start clean
  return e == cudaErrorMemoryAllocation ? ARMT_ERR_OOM : ARMT_ERR_CUDA;
}

#define ARMT_TRY(call, where)                         \
  do {                                                \
    cudaError_t e_ = (call);                          \
    if (e_ != cudaSuccess) return cuda_fail(ctx, e_, where); \
  } while (0)

size_t act_size(const Dims& dm) { return dm.bf16 ? 2 : 4; }

template <typename T>
cudaError_t dalloc(T** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) return cudaSuccess;
  return cudaMalloc((void**)p, bytes);
}

void dfree(void* p) {
  if (p) cudaFree(p);
}

void free_weights(Weights& w) {
  dfree(w.mem_emb); dfree(w.w_qkv); dfree(w.w_o); dfree(w.w_gu); dfree(w.w_down);
  dfree(w.w_qm); dfree(w.w_kvm);
  w = Weights();
}

void free_workspace(Workspace& ws) {
  dfree(ws.h); dfree(ws.xb); dfree(ws.qm); dfree(ws.phi); dfree(ws.inv_den); dfree(ws.qkv);
  dfree(ws.attn); dfree(ws.gu); dfree(ws.u); dfree(ws.kv); dfree(ws.phik); dfree(ws.coef);
  dfree(ws.gamma); dfree(ws.beta); dfree(ws.rope); dfree(ws.nodes); dfree(ws.err); dfree(ws.rsq); dfree(ws.gram); dfree(ws.vt);
  ws = Workspace();
}

armt_status validate_config(const armt_config* c, const char** why) {
  if (!c) { *why = "null config"; return ARMT_ERR_INVALID_ARG; }
  if (c->n_layers < 1 || c->d_model < 1 || c->n_heads < 1 || c->n_kv_heads < 1 || c->head_dim < 2 ||
      c->d_ffn < 1 || c->n_mem < 0 || c->d_key < 1 || c->dpfp_nu < 1 || c->max_seg_len < 1 ||
      c->max_segments < 1) {
    *why = "every size must be positive"; return ARMT_ERR_INVALID_ARG;
  }
  if (c->n_heads % c->n_kv_heads) { *why = "n_heads must be a multiple of n_kv_heads"; return ARMT_ERR_INVALID_ARG; }
  if (c->head_dim % 2) { *why = "head_dim must be even"; return ARMT_ERR_INVALID_ARG; }
  if (c->dtype != ARMT_FP32 && c->dtype != ARMT_BF16) { *why = "unknown dtype"; return ARMT_ERR_INVALID_ARG; }
  if (c->schedule != ARMT_SCHED_DIAGONAL && c->schedule != ARMT_SCHED_SEQUENTIAL) {
    *why = "unknown schedule"; return ARMT_ERR_INVALID_ARG;
  }
  if (!(c->rms_eps >= 0.f) || !(c->mem_eps > 0.f) || !(c->rope_theta > 0.f)) {
    *why = "eps must be >= 0 (rms) / > 0 (memory), rope_theta > 0"; return ARMT_ERR_INVALID_ARG;
  }
  if (c->dpfp_nu > 2 * c->d_key) { *why = "dpfp_nu must be <= 2 * d_key"; return ARMT_ERR_INVALID_ARG; }
  if ((c->write_gate != 0 && c->write_gate != 1) || (c->gamma_unclamped != 0 && c->gamma_unclamped != 1)) {
    *why = "write_gate and gamma_unclamped must be 0 or 1"; return ARMT_ERR_INVALID_ARG;
  }
  if (c->head_dim != 16 && c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128) {
    *why = "head_dim must be 16, 32, 64 or 128"; return ARMT_ERR_UNSUPPORTED;
  }
  const long long P = 2LL * c->d_key * c->dpfp_nu;
  if (P > 1024) { *why = "phi dimension 2*d_key*nu must be <= 1024"; return ARMT_ERR_UNSUPPORTED; }
  if (c->n_mem > 32) { *why = "n_mem must be <= 32"; return ARMT_ERR_UNSUPPORTED; }
  if (((long long)c->n_mem * P + (long long)c->n_mem * c->n_mem + 17LL * c->n_mem) * 4 > 200 * 1024 ||
      ((long long)P + (long long)c->n_mem * P + (long long)(c->n_mem < 32 ? c->n_mem : 32) * 2 * c->d_key +
       2LL * c->n_mem + (long long)c->n_mem * c->n_mem) * 4 > 200 * 1024) {
    *why = "n_mem * phi dimension too large for the write kernel"; return ARMT_ERR_UNSUPPORTED;
  }
  if (c->dtype == ARMT_BF16 && (c->d_model % 8 || c->d_ffn % 8 || (c->n_heads * c->head_dim) % 8 || P % 8)) {
    *why = "bf16 mode needs d_model, d_ffn, H*hd and phi dimension multiples of 8"; return ARMT_ERR_UNSUPPORTED;
  }
  if (c->dtype == ARMT_BF16 && c->head_dim != 64 && c->head_dim != 128) {
    *why = "bf16 mode needs head_dim 64 or 128"; return ARMT_ERR_UNSUPPORTED;
  }
  return ARMT_OK;
}

// Node table for (S, schedule): entries in launch order, grouped into waves.
// The wave made of table entries first .. end (layers 0 .. L-1 of the context).
Wave summarize_wave(const std::vector<NodeEntry>& tab, int first, int L) {
  Wave w;
  w.first = first;
  w.count = (int)tab.size() - first;
  w.any_first_layer = false;
  w.any_last_layer = false;
  w.first_layer_pos = -1;
  w.first_layer_seg = -1;
  w.last_layer_seg = -1;
  for (int k = first; k < (int)tab.size(); ++k) {
    if (tab[k].y == 0) {   // a wave holds at most one layer-0 node
      w.first_layer_pos = k - first;
      w.first_layer_seg = tab[k].x;
    }
    if (tab[k].y == L - 1) w.last_layer_seg = tab[k].x;   // and at most one last-layer node
    w.any_first_layer |= tab[k].y == 0;
    w.any_last_layer |= tab[k].y == L - 1;
  }
  return w;
}

void build_table(int S, int L, int slots, armt_schedule sched, std::vector<NodeEntry>& tab,
                 std::vector<Wave>& waves) {
  tab.clear();
  waves.clear();
  auto push_wave = [&](int first) { waves.push_back(summarize_wave(tab, first, L)); };
  if (sched == ARMT_SCHED_DIAGONAL) {
    for (int i = 0; i < S + L - 1; ++i) {
      const int first = (int)tab.size();
      for (int l = std::max(0, i - S + 1); l <= std::min(i, L - 1); ++l) {
        const int s = i - l;
        tab.push_back(make_int4(s, l, s % slots, 0));
      }
      push_wave(first);
    }
  } else {
    for (int s = 0; s < S; ++s)
      for (int l = 0; l < L; ++l) {
        const int first = (int)tab.size();
        tab.push_back(make_int4(s, l, s % slots, 0));
        push_wave(first);
      }
  }
}

// Layer-pipeline stage holding global layers offset .. offset + L - 1 of a
// model of `total` layers: one entry per global wave i = 0 .. S + total - 2
// (possibly empty), with the nodes (s, j) of local layer j = l - offset,
// s = i - l, 0 <= s < S.
void build_stage_table(int S, int L, int offset, int total, int slots, std::vector<NodeEntry>& tab,
                       std::vector<Wave>& waves) {
  tab.clear();
  waves.clear();
  for (int i = 0; i < S + total - 1; ++i) {
    const int first = (int)tab.size();
    for (int j = 0; j < L; ++j) {
      const int s = i - offset - j;
      if (s >= 0 && s < S) tab.push_back(make_int4(s, j, s % slots, 0));
    }
    waves.push_back(summarize_wave(tab, first, L));
  }
}

// Kernel kinds, in the order a wave launches them (both paths).
const char* const KIND_NAMES[] = {
    "init", "gemm_qmem", "tc_qmem", "dpfp_read", "gemm_read", "tc_read", "norm_attn", "gemm_qkv",
    "rope", "tc_qkv_rope", "attention", "gemm_o", "tc_o", "norm_mlp", "gemm_gateup", "swiglu",
    "tc_gateup_swiglu", "gemm_down", "tc_down", "norm_mem", "gemm_kvmem", "tc_kvmem", "memw_phi", "memw_update",
    "output"};
constexpr int N_KINDS = (int)(sizeof(KIND_NAMES) / sizeof(KIND_NAMES[0]));

int kind_index(const char* name) {
  for (int k = 0; k < N_KINDS; ++k)
    if (!strcmp(KIND_NAMES[k], name)) return k;
  return -1;
}

struct Launcher {
  bool dry = false;
  int count = 0;
  cudaError_t err = cudaSuccess;
  const char* where = "";
  // profiling: events around every launch on the launching stream
  bool profile = false;
  cudaStream_t pstream = nullptr;
  std::vector<cudaEvent_t> ev;
  std::vector<int> kinds;
  template <typename F>
  void operator()(const char* name, F&& f) {
    ++count;
    if (dry || err != cudaSuccess) return;
    if (profile) {
      cudaEvent_t a, b;
      err = cudaEventCreate(&a);
      if (err == cudaSuccess) err = cudaEventCreate(&b);
      if (err != cudaSuccess) { where = "event create"; return; }
      ev.push_back(a);
      ev.push_back(b);
      kinds.push_back(kind_index(name));
      cudaEventRecord(a, pstream);
      err = f();
      cudaEventRecord(b, pstream);
    } else {
      err = f();
    }
    if (err != cudaSuccess) where = name;
  }
  ~Launcher() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
  }
};

// fp32 path: enqueue every kernel of one wave (SIMT kernels, fp32 throughout).
// T = seg_len, Tp = T + M rows per node.
// stage_in / stage_out: layer-pipeline hand-off rows (null in a whole forward).
void enqueue_wave(armt_ctx* ctx, const Wave& wv, int T, const void* emb, void* out, float* A, float* z,
                  cudaStream_t st, Launcher& L, const float* stage_in = nullptr, float* stage_out = nullptr) {
  const Dims& dm = ctx->dm;
  Workspace& ws = ctx->ws;
  const Weights& w = ctx->w;
  const int Tp = T + dm.M;
  const int n = wv.count;
  const NodeEntry* nodes = ws.nodes + wv.first;
  const long long hs = (long long)Tp * dm.d;
  void* a_read = A;

  if (wv.any_first_layer)
    L("init", [&] {   // only the wave's layer-0 node
      if (stage_in)
        return launch_stage_rows_in(dm, nodes + wv.first_layer_pos, 1, 0, Tp, stage_in, ws.h, nullptr, st);
      return launch_init_first_layer(dm, nodes + wv.first_layer_pos, 1, T, Tp, emb, w.mem_emb, ws.h, nullptr, st);
    });

  // ---- memory read: q = h Wq_mem^T, phi = DPFP(q), h += phi A^T / (z.phi + eps)
  // (no memory tokens: no associative memory, the layer alone)
  if (dm.M > 0) {
    GemmArgs g{};
    g.nodes = nodes; g.n_nodes = n; g.M = Tp; g.N = dm.dk; g.K = dm.d;
    g.A = ws.h; g.a_slot_stride = hs; g.lda = dm.d;
    g.B = w.w_qm; g.b_layer_stride = (long long)dm.dk * dm.d; g.ldb = dm.d;
    g.C = ws.qm; g.c_slot_stride = (long long)Tp * dm.dk; g.ldc = dm.dk;
    g.epi = EPI_STORE_F32;
    L("gemm_qmem", [&] { return launch_simt_gemm(g, st); });
  }
  if (dm.M > 0) L("dpfp_read", [&] { return launch_dpfp_read(dm, nodes, n, Tp, ws.qm, z, ws.phi, ws.inv_den, st); });
  if (dm.M > 0) {
    GemmArgs g{};
    g.nodes = nodes; g.n_nodes = n; g.M = Tp; g.N = dm.d; g.K = dm.P;
    g.A = ws.phi; g.a_slot_stride = (long long)Tp * dm.P; g.lda = dm.P;
    g.B = a_read; g.b_layer_stride = (long long)dm.d * dm.P; g.ldb = dm.P;
    g.C = ws.h; g.c_slot_stride = hs; g.ldc = dm.d;
    g.rowscale = ws.inv_den; g.rs_slot_stride = Tp;
    g.epi = EPI_RESID;
    L("gemm_read", [&] { return launch_simt_gemm(g, st); });
  }

  // ---- attention block
  L("norm_attn", [&] { return launch_rmsnorm(dm, nodes, n, Tp, 0, Tp, ws.h, ws.xb, dm.rms_eps, st); });
  {
    GemmArgs g{};
    g.nodes = nodes; g.n_nodes = n; g.M = Tp; g.N = dm.nqkv; g.K = dm.d;
    g.A = ws.xb; g.a_slot_stride = hs; g.lda = dm.d;
    g.B = w.w_qkv; g.b_layer_stride = (long long)dm.nqkv * dm.d; g.ldb = dm.d;
    g.C = ws.qkv; g.c_slot_stride = (long long)Tp * dm.nqkv; g.ldc = dm.nqkv;
    g.epi = EPI_STORE_ACT;
    L("gemm_qkv", [&] { return launch_simt_gemm(g, st); });
  }
  L("rope", [&] { return launch_rope(dm, nodes, n, Tp, ws.qkv, ws.rope, ws.tp_max, st); });
  L("attention", [&] { return launch_attention_simt(dm, nodes, n, Tp, ws.qkv, ws.attn, st); });
  {
    GemmArgs g{};
    g.nodes = nodes; g.n_nodes = n; g.M = Tp; g.N = dm.d; g.K = dm.H * dm.hd;
    g.A = ws.attn; g.a_slot_stride = (long long)Tp * dm.H * dm.hd; g.lda = dm.H * dm.hd;
    g.B = w.w_o; g.b_layer_stride = (long long)dm.d * dm.H * dm.hd; g.ldb = dm.H * dm.hd;
    g.C = ws.h; g.c_slot_stride = hs; g.ldc = dm.d;
    g.epi = EPI_RESID;
    L("gemm_o", [&] { return launch_simt_gemm(g, st); });
  }

  // ---- MLP block
  L("norm_mlp", [&] { return launch_rmsnorm(dm, nodes, n, Tp, 0, Tp, ws.h, ws.xb, dm.rms_eps, st); });
  {
    GemmArgs g{};
    g.nodes = nodes; g.n_nodes = n; g.M = Tp; g.N = 2 * dm.F; g.K = dm.d;
    g.A = ws.xb; g.a_slot_stride = hs; g.lda = dm.d;
    g.B = w.w_gu; g.b_layer_stride = 2LL * dm.F * dm.d; g.ldb = dm.d;
    g.C = ws.gu; g.c_slot_stride = 2LL * Tp * dm.F; g.ldc = 2 * dm.F;
    g.epi = EPI_STORE_ACT;
    L("gemm_gateup", [&] { return launch_simt_gemm(g, st); });
  }
  L("swiglu", [&] { return launch_swiglu(dm, nodes, n, Tp, ws.gu, ws.u, st); });
  {
    GemmArgs g{};
    g.nodes = nodes; g.n_nodes = n; g.M = Tp; g.N = dm.d; g.K = dm.F;
    g.A = ws.u; g.a_slot_stride = (long long)Tp * dm.F; g.lda = dm.F;
    g.B = w.w_down; g.b_layer_stride = (long long)dm.d * dm.F; g.ldb = dm.F;
    g.C = ws.h; g.c_slot_stride = hs; g.ldc = dm.d;
    g.epi = EPI_RESID;
    L("gemm_down", [&] { return launch_simt_gemm(g, st); });
  }

  // ---- memory write from the RMS-normalised M memory rows of the layer output
  if (dm.M > 0) L("norm_mem", [&] { return launch_rmsnorm(dm, nodes, n, Tp, T, dm.M, ws.h, ws.xb, dm.rms_eps, st); });
  if (dm.M > 0) {
    const int ldkv = kv_ld(dm);
    GemmArgs g{};
    g.nodes = nodes; g.n_nodes = n; g.M = dm.M; g.N = ldkv; g.K = dm.d;
    g.A = (const float*)ws.xb + (long long)T * dm.d; g.a_slot_stride = hs; g.lda = dm.d;
    g.B = w.w_kvm; g.b_layer_stride = (long long)ldkv * dm.d; g.ldb = dm.d;
    g.C = ws.kv; g.c_slot_stride = (long long)dm.M * ldkv; g.ldc = ldkv;
    g.epi = EPI_STORE_F32;
    L("gemm_kvmem", [&] { return launch_simt_gemm(g, st); });
  }
  if (dm.M > 0) {
    L("memw_phi", [&] {
      return launch_memw_phi(dm, nodes, n, ws.kv, z, ws.phik, ws.gram, ws.coef, ws.gamma, ws.beta, st);
    });
    L("memw_update", [&] {
      return launch_memw_update(dm, nodes, n, ws.kv, ws.phik, ws.gram, ws.coef, ws.beta, A, st);
    });
  }

  if (wv.any_last_layer && stage_out)
    L("output", [&] { return launch_stage_rows_out(dm, nodes, n, dm.L - 1, Tp, ws.h, stage_out, st); });
  else if (wv.any_last_layer)
    L("output", [&] { return launch_output(dm, nodes, n, T, Tp, ws.h, out, st); });
}

// Column tile of the memory-write projection (16 rows per node, weight-read
// bound: narrower tiles put more CTAs, so more weight loads, in flight);
// ARMT_KVMEM_BN selects 64 / 128 / 256 for measurement.
int kvmem_bn() {
  static const int bn = [] {
    const char* v = getenv("ARMT_KVMEM_BN");
    const int b = v ? atoi(v) : 256;
    return (b == 64 || b == 128) ? b : 256;
  }();
  return bn;
}

// The memory write of a wave (projection, features, update of A and z) runs on
// a second stream, so that the next wave's first kernels overlap it: the
// memory-read query of wave i+1 needs only the layer outputs of wave i; the
// DPFP read needs z (written by the feature kernel); the read product needs
// A (written by the update).  The layer-0 input of wave i+1 overwrites a slot
// whose memory rows wave i's projection reads (wave i holds every slot), so
// it waits for that projection.  Each wait is an event on the previous wave's
// write; nothing waits when there is none yet.
struct WriteOverlap {
  cudaStream_t s2;
  cudaEvent_t down, kv, phi, upd;   // recorded after: down GEMM (s1); projection, features, update (s2)
  bool pending = false;              // a wave's write was enqueued and not yet joined
};

// Tensor-core path (bf16 mode): the dense products run on the tcgen05 grouped
// GEMM with fused epilogues, attention on tensor cores.  Weights hold the
// bf16-rounded values in fp16 containers and the GEMM activations are fp16
// (same tensor-core rate as bf16, 3 more mantissa bits: rounding the
// normalised activations to bf16 alone costs ~1 % relative error over 16
// layers).  The memory read multiplies the fp32 features and the fp32 state
// A itself at tf32 precision (fp16's mantissa, fp32's range), so no copy of
// A is kept.  Residual stream, accumulation and the memory state are fp32.
void enqueue_wave_tc(armt_ctx* ctx, const Wave& wv, int T, const void* emb, void* out, float* A, float* z,
                     cudaStream_t st, Launcher& L, WriteOverlap* ov = nullptr, const float* stage_in = nullptr,
                     float* stage_out = nullptr) {
  const Dims& dm = ctx->dm;
  Workspace& ws = ctx->ws;
  const Weights& w = ctx->w;
  const int Tp = T + dm.M;
  const int n = wv.count;
  const NodeEntry* nodes = ws.nodes + wv.first;
  const int slots = ws.slots;
  const long long hs = (long long)Tp * dm.d;
  const long long hs_blk = (long long)rows_blocked(Tp) * dm.d;   // row-blocked residual, per slot
  const int Hh = dm.H * dm.hd;
  const int f_pad = (dm.F + 127) / 128 * 128;
  const int sms = ctx->sm_count;
  auto base = [&](TcGemmParams& p, int M, int N, int K) {
    p = TcGemmParams{};
    p.nodes = nodes; p.n_nodes = n; p.M = M; p.N = N; p.K = K; p.err = ws.err;
    p.out_layer = -1;
  };
  const int rsq_parts = 2 * ((dm.d + 255) / 256);   // one partial per half of a 256-column tile
  auto norm_partials = [&](TcGemmParams& p) {
    p.rsq = ws.rsq; p.rsq_slot_stride = (long long)Tp * rsq_parts; p.rsq_parts = rsq_parts; p.rsq_pitch = Tp;
    p.norm_dim = dm.d; p.norm_eps = dm.rms_eps;
  };
  // stream s waits for event e of the previous wave's write (no-op without one)
  auto after = [&](cudaStream_t s, cudaEvent_t e) {
    if (ov && ov->pending && !L.dry && L.err == cudaSuccess) {
      L.err = cudaStreamWaitEvent(s, e, 0);
      if (L.err != cudaSuccess) L.where = "stream wait";
    }
  };
  auto mark = [&](cudaEvent_t e, cudaStream_t s) {
    if (ov && !L.dry && L.err == cudaSuccess) {
      L.err = cudaEventRecord(e, s);
      if (L.err != cudaSuccess) L.where = "event record";
    }
  };

  if (wv.any_first_layer) {
    if (ov) after(st, ov->kv);
    L("init", [&] {   // only the wave's layer-0 node
      if (stage_in)
        return launch_stage_rows_in(dm, nodes + wv.first_layer_pos, 1, 0, Tp, stage_in, ws.h, ws.xb, st);
      return launch_init_first_layer(dm, nodes + wv.first_layer_pos, 1, T, Tp, emb, w.mem_emb, ws.h, (f16*)ws.xb, st);
    });
  }
  // no memory tokens: no associative memory.  The QKV epilogue's RMSNorm row
  // scale then needs the layer-0 input's sums of squares, which the memory
  // read's residual epilogue would otherwise have written.
  if (dm.M == 0 && wv.any_first_layer)
    L("init", [&] {
      return launch_row_sumsq(dm, nodes + wv.first_layer_pos, 1, Tp, ws.h, ws.rsq, (long long)Tp * rsq_parts,
                              rsq_parts, Tp, st);
    });

  // ---- memory read
  if (dm.M > 0) {
  L("tc_qmem", [&] {
    TcGemmOperands op{ws.xb, Tp, slots, w.w_qm, dm.dk, dm.L};
    TcGemmParams p; base(p, Tp, dm.dk, dm.d);
    p.C = ws.qm; p.c_slot_stride = (long long)Tp * dm.dk; p.ldc = dm.dk;
    return launch_tc_gemm(op, p, TC_EPI_F32, tc_pick_bn(dm.dk), sms, st);
  });
  if (ov) after(st, ov->phi);
  L("dpfp_read", [&] { return launch_dpfp_read(dm, nodes, n, Tp, ws.qm, z, ws.phi, ws.inv_den, st); });
  if (ov) after(st, ov->upd);
  L("tc_read", [&] {
    // h += phi A^T / (z.phi + eps) on kind::tf32 (phi and A fp32); new h ->
    // fp16 operand copy + norm partials
    TcGemmOperands op{ws.phi, Tp, slots, A, dm.d, dm.L};
    TcGemmParams p; base(p, Tp, dm.d, dm.P);
    p.ab_tf32 = 1;
    p.h = ws.h; p.h_slot_stride = hs_blk; p.ldh = dm.d;
    p.rowscale = ws.inv_den; p.rs_slot_stride = Tp;
    p.C = ws.xb; p.c_slot_stride = hs; p.ldc = dm.d;
    norm_partials(p);
    return launch_tc_gemm(op, p, TC_EPI_RESID_ACT, 256, sms, st);
  });
  }

  // ---- attention block (RMSNorm folded: row scale applied in the QKV epilogue)
  L("tc_qkv_rope", [&] {
    TcGemmOperands op{ws.xb, Tp, slots, w.w_qkv, dm.nqkv, dm.L};
    TcGemmParams p; base(p, Tp, dm.nqkv, dm.d);
    p.C = ws.qkv; p.c_slot_stride = (long long)Tp * dm.nqkv; p.ldc = dm.nqkv;
    p.rope = ws.rope; p.rope_pitch = ws.tp_max; p.rope_heads = dm.H + dm.KV; p.head_dim = dm.hd;
    if (ws.vt) {
      p.vt = (f16*)ws.vt; p.vt_pitch = attention_tc_vt_pitch(Tp); p.n_vheads = dm.KV;
    }
    norm_partials(p);
    return launch_tc_gemm(op, p, TC_EPI_QKV_ROPE, 256, sms, st);
  });
  L("attention", [&] { return launch_attention_tc(dm, nodes, n, Tp, slots, ws.qkv, ws.vt, ws.attn, ws.err, st); });
  L("tc_o", [&] {
    TcGemmOperands op{ws.attn, Tp, slots, w.w_o, dm.d, dm.L};
    TcGemmParams p; base(p, Tp, dm.d, Hh);
    p.h = ws.h; p.h_slot_stride = hs_blk; p.ldh = dm.d;
    p.C = ws.xb; p.c_slot_stride = hs; p.ldc = dm.d;
    norm_partials(p);
    return launch_tc_gemm(op, p, TC_EPI_RESID_ACT, 256, sms, st);
  });

  // ---- MLP block (RMSNorm folded into the gate/up epilogue)
  L("tc_gateup_swiglu", [&] {
    TcGemmOperands op{ws.xb, Tp, slots, w.w_gu, 2 * f_pad, dm.L};
    TcGemmParams p; base(p, Tp, 2 * f_pad, dm.d);
    p.C = ws.u; p.c_slot_stride = (long long)Tp * dm.F; p.ldc = dm.F; p.f_out = dm.F;
    norm_partials(p);
    return launch_tc_gemm(op, p, TC_EPI_SWIGLU, 256, sms, st);
  });
  L("tc_down", [&] {
    // h += u W_d^T; new h -> fp16 copy (next layer's memory-read query and
    // this node's memory-write rows); last layer: rows < T -> out_hidden
    TcGemmOperands op{ws.u, Tp, slots, w.w_down, dm.d, dm.L};
    TcGemmParams p; base(p, Tp, dm.d, dm.F);
    p.h = ws.h; p.h_slot_stride = hs_blk; p.ldh = dm.d;
    p.C = ws.xb; p.c_slot_stride = hs; p.ldc = dm.d;
    p.out = out; p.out_layer = dm.L - 1; p.seg_len = T;
    norm_partials(p);   // for the memory-write rows
    return launch_tc_gemm(op, p, TC_EPI_RESID_ACT, 256, sms, st);
  });
  // layer pipeline: this stage's last layer hands its rows to the next stage
  if (stage_out && wv.any_last_layer)
    L("output", [&] { return launch_stage_rows_out(dm, nodes, n, dm.L - 1, Tp, ws.h, stage_out, st); });

  // ---- memory write: [k | v] = RMSNorm(m) [Wk_mem; Wv_mem]^T for the M memory
  // rows (rows T..T'-1 of the fp16 copy of the layer output the down GEMM
  // wrote; the RMS row scale comes from the down GEMM's partial sums)
  if (dm.M == 0) return;
  cudaStream_t cs = st;   // the write's stream
  if (ov) {
    mark(ov->down, st);
    if (!L.dry && L.err == cudaSuccess) {
      L.err = cudaStreamWaitEvent(ov->s2, ov->down, 0);
      if (L.err != cudaSuccess) L.where = "stream wait";
    }
    cs = ov->s2;
  }
  L("tc_kvmem", [&] {
    const int ldkv = kv_ld(dm);
    TcGemmOperands op{(const char*)ws.xb + (size_t)T * dm.d * 2, dm.M, slots, w.w_kvm, ldkv, dm.L};
    op.a_pitch = Tp;
    TcGemmParams p; base(p, dm.M, ldkv, dm.d);
    p.C = ws.kv; p.c_slot_stride = (long long)dm.M * ldkv; p.ldc = ldkv;
    norm_partials(p);
    p.rsq_row0 = T;
    return launch_tc_gemm(op, p, TC_EPI_F32, kvmem_bn(), sms, cs);
  });
  if (ov) mark(ov->kv, cs);
  L("memw_phi", [&] {
    return launch_memw_phi(dm, nodes, n, ws.kv, z, ws.phik, ws.gram, ws.coef, ws.gamma, ws.beta, cs);
  });
  if (ov) mark(ov->phi, cs);
  L("memw_update", [&] {
    return launch_memw_update(dm, nodes, n, ws.kv, ws.phik, ws.gram, ws.coef, ws.beta, A, cs);
  });
  if (ov) {
    mark(ov->upd, cs);
    ov->pending = true;
  }
}

// Ties the last wave's write back into stream st.
cudaError_t join_write(WriteOverlap* ov, cudaStream_t st) {
  if (!ov || !ov->pending) return cudaSuccess;
  ov->pending = false;
  return cudaStreamWaitEvent(st, ov->upd, 0);
}

armt_status ensure_table(armt_ctx* ctx, int S, cudaStream_t st) {
  const armt_schedule sched = ctx->cfg.schedule;
  if (ctx->table_S == S && ctx->table_sched == (int)sched) return ARMT_OK;
  std::vector<NodeEntry> tab;
  build_table(S, ctx->dm.L, ctx->ws.slots, sched, tab, ctx->waves);
  if ((int)tab.size() > ctx->ws.nodes_cap) return fail(ctx, ARMT_ERR_SHAPE, "node table too large");
  ARMT_TRY(cudaMemcpyAsync(ctx->ws.nodes, tab.data(), tab.size() * sizeof(NodeEntry),
                           cudaMemcpyHostToDevice, st), "upload node table");
  ARMT_TRY(cudaStreamSynchronize(st), "upload node table");
  ctx->table_S = S;
  ctx->table_sched = (int)sched;
  ctx->stage_S = -1;   // the stage table (same device buffer) is gone
  return ARMT_OK;
}

// The write overlap of the tensor-core path (streams and events created once).
WriteOverlap* write_overlap(armt_ctx* ctx) {
  if (!ctx->ov_stream) {
    if (cudaStreamCreateWithFlags(&ctx->ov_stream, cudaStreamNonBlocking) != cudaSuccess) {
      cudaGetLastError();
      ctx->ov_stream = nullptr;
      return nullptr;
    }
    for (cudaEvent_t* e : {&ctx->ov_ev[0], &ctx->ov_ev[1], &ctx->ov_ev[2], &ctx->ov_ev[3]})
      if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
      }
  }
  static thread_local WriteOverlap ov;
  ov.s2 = ctx->ov_stream;
  ov.down = ctx->ov_ev[0]; ov.kv = ctx->ov_ev[1]; ov.phi = ctx->ov_ev[2]; ov.upd = ctx->ov_ev[3];
  ov.pending = false;
  return &ov;
}

// carry_state: A and z already hold the state to start from (else zeroed first).
// overlap: run each wave's memory write on the second stream (tensor-core path;
// not in the per-kernel profile, whose events time one stream).
armt_status enqueue_forward(armt_ctx* ctx, const void* emb, int S, int T, void* out, float* A, float* z,
                            cudaStream_t st, Launcher& L, bool carry_state = false, bool overlap = false) {
  const Dims& dm = ctx->dm;
  if (!L.dry && !carry_state) {
    ARMT_TRY(cudaMemsetAsync(A, 0, (size_t)dm.L * dm.d * dm.P * sizeof(float), st), "zero A");
    ARMT_TRY(cudaMemsetAsync(z, 0, (size_t)dm.L * dm.P * sizeof(float), st), "zero z");
  }
  WriteOverlap* ov = (overlap && dm.bf16 && dm.M > 0 && !L.dry && !L.profile) ? write_overlap(ctx) : nullptr;
  for (const Wave& wv : ctx->waves) {
    if (dm.bf16) enqueue_wave_tc(ctx, wv, T, emb, out, A, z, st, L, ov);
    else enqueue_wave(ctx, wv, T, emb, out, A, z, st, L);
    if (L.err != cudaSuccess) return cuda_fail(ctx, L.err, L.where);
  }
  ARMT_TRY(join_write(ov, st), "join the memory write");
  return ARMT_OK;
}

armt_status check_forward_args(armt_ctx* ctx, const void* emb, int S, int seg_len, const void* out,
                               const float* A, const float* z) {
  if (!ctx) return ARMT_ERR_INVALID_ARG;
  if (!emb || !out || !A || !z) return fail(ctx, ARMT_ERR_INVALID_ARG, "null buffer");
  if (S < 1 || seg_len < 1) return fail(ctx, ARMT_ERR_INVALID_ARG, "S and seg_len must be >= 1");
  if (!ctx->w.loaded) return fail(ctx, ARMT_ERR_NOT_LOADED, "weights not loaded");
  if (S > ctx->cfg.max_segments) return fail(ctx, ARMT_ERR_SHAPE, "S > max_segments");
  if (seg_len > ctx->cfg.max_seg_len) return fail(ctx, ARMT_ERR_SHAPE, "seg_len > max_seg_len");
  return ARMT_OK;
}

armt_status forward_impl(armt_ctx* ctx, const void* emb, int S, int T, void* out, float* A, float* z,
                         cudaStream_t st, bool carry_state = false) {
  armt_status s = ensure_table(ctx, S, st);
  if (s != ARMT_OK) return s;
  if (!ctx->use_graph) {
    Launcher L;
    return enqueue_forward(ctx, emb, S, T, out, A, z, st, L, carry_state, ctx->overlap_write);
  }
  armt_ctx::GraphKey key;
  key.S = S; key.T = T; key.sched = (int)ctx->cfg.schedule; key.carry = carry_state ? 1 : 0;
  key.emb = emb; key.out = out; key.A = A; key.z = z;
  const armt_ctx::GraphKey& k0 = ctx->graph_key;
  const bool same = ctx->graph_exec && k0.S == key.S && k0.T == key.T && k0.sched == key.sched &&
                    k0.carry == key.carry && k0.emb == key.emb && k0.out == key.out && k0.A == key.A &&
                    k0.z == key.z;
  if (!same) {
    if (ctx->graph_exec) {
      cudaGraphExecDestroy(ctx->graph_exec);
      ctx->graph_exec = nullptr;
    }
    ARMT_TRY(cudaStreamBeginCapture(ctx->capture_stream, cudaStreamCaptureModeThreadLocal), "begin capture");
    Launcher L;
    armt_status es = enqueue_forward(ctx, emb, S, T, out, A, z, ctx->capture_stream, L, carry_state,
                                     ctx->overlap_write);
    cudaGraph_t graph = nullptr;
    cudaError_t ce = cudaStreamEndCapture(ctx->capture_stream, &graph);
    if (es != ARMT_OK) {
      if (graph) cudaGraphDestroy(graph);
      return es;
    }
    if (ce != cudaSuccess) return cuda_fail(ctx, ce, "end capture");
    ce = cudaGraphInstantiate(&ctx->graph_exec, graph, 0);
    cudaGraphDestroy(graph);
    if (ce != cudaSuccess) {
      ctx->graph_exec = nullptr;
      return cuda_fail(ctx, ce, "graph instantiate");
    }
    ctx->graph_key = key;
  }
  ARMT_TRY(cudaGraphLaunch(ctx->graph_exec, st), "graph launch");
  return ARMT_OK;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================

extern "C" const char* armt_status_string(armt_status s) {
  switch (s) {
    case ARMT_OK: return "ok";
    case ARMT_ERR_INVALID_ARG: return "invalid argument";
    case ARMT_ERR_NOT_LOADED: return "weights not loaded";
    case ARMT_ERR_SHAPE: return "shape exceeds the context's maxima";
    case ARMT_ERR_OOM: return "device out of memory";
    case ARMT_ERR_CUDA: return "CUDA error";
    case ARMT_ERR_DEVICE_TIMEOUT: return "device-side bounded wait timed out";
    case ARMT_ERR_UNSUPPORTED: return "unsupported shape";
    case ARMT_ERR_NUMERIC_RANGE: return "numeric range (reserved)";
  }
  return "unknown status";
}

extern "C" const char* armt_last_error(armt_ctx* ctx) {
  return ctx ? ctx->last_error.c_str() : "null context";
}

extern "C" armt_status armt_create(const armt_config* cfg, armt_ctx** out) {
  if (!out) return ARMT_ERR_INVALID_ARG;
  *out = nullptr;
  const char* why = "";
  armt_status vs = validate_config(cfg, &why);
  if (vs != ARMT_OK) return vs;
  armt_ctx* ctx = new armt_ctx();
  ctx->cfg = *cfg;
  {
    const char* v = getenv("ARMT_OVERLAP_WRITE");   // "0": memory write in line (A/B measurement)
    ctx->overlap_write = !(v && v[0] == '0');
  }
  Dims& dm = ctx->dm;
  dm.L = cfg->n_layers; dm.d = cfg->d_model; dm.H = cfg->n_heads; dm.KV = cfg->n_kv_heads;
  dm.hd = cfg->head_dim; dm.F = cfg->d_ffn; dm.M = cfg->n_mem; dm.dk = cfg->d_key; dm.nu = cfg->dpfp_nu;
  dm.P = 2 * dm.dk * dm.nu; dm.nqkv = (dm.H + 2 * dm.KV) * dm.hd;
  dm.theta = cfg->rope_theta; dm.rms_eps = cfg->rms_eps; dm.mem_eps = cfg->mem_eps;
  dm.bf16 = cfg->dtype == ARMT_BF16;
  dm.write_gate = cfg->write_gate != 0;
  dm.clamp_gamma = cfg->gamma_unclamped == 0;

  cudaError_t e = cudaGetDevice(&ctx->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&ctx->sm_count, cudaDevAttrMultiProcessorCount, ctx->device);
  if (e != cudaSuccess) {
    armt_status s = cuda_fail(nullptr, e, "device");
    delete ctx;
    return s;
  }
  Workspace& ws = ctx->ws;
  ws.slots = std::min(cfg->max_segments, dm.L);
  ws.tp_max = cfg->max_seg_len + dm.M;
  const size_t rows = (size_t)ws.slots * ws.tp_max;
  const size_t as = act_size(dm);
  const size_t ntab = (size_t)cfg->max_segments * dm.L;
  e = cudaSuccess;
  auto A = [&](auto** p, size_t bytes) { if (e == cudaSuccess) e = dalloc(p, bytes); };
  A(&ws.h, (size_t)ws.slots * rows_blocked(ws.tp_max) * dm.d * 4);   // >= rows * d (row-blocked slots)
  A(&ws.xb, rows * dm.d * as);
  A(&ws.qm, rows * dm.dk * 4);
  A(&ws.phi, rows * dm.P * 4);
  A(&ws.inv_den, rows * 4);
  if (dm.bf16) A(&ws.rsq, rows * 2 * ((dm.d + 255) / 256) * 4);
  A(&ws.qkv, rows * dm.nqkv * as);
  A(&ws.attn, rows * dm.H * dm.hd * as);
  if (dm.bf16 && attention_tc_supported(dm))
    A(&ws.vt, (size_t)ws.slots * dm.KV * dm.hd * attention_tc_vt_pitch(ws.tp_max) * 2);
  if (!dm.bf16) A(&ws.gu, rows * 2 * dm.F * as);
  A(&ws.u, rows * dm.F * as);
  A(&ws.kv, (size_t)ws.slots * dm.M * kv_ld(dm) * 4);
  A(&ws.phik, (size_t)ws.slots * dm.M * dm.P * 4);
  A(&ws.coef, (size_t)ws.slots * dm.M * 4);
  A(&ws.gram, (size_t)ws.slots * dm.M * dm.M * 4);
  A(&ws.gamma, (size_t)ws.slots * dm.M * 4);
  A(&ws.beta, (size_t)ws.slots * dm.M * 4);
  A(&ws.rope, (size_t)ws.tp_max * (dm.hd / 2) * sizeof(float2));
  A(&ws.nodes, ntab * sizeof(NodeEntry));
  A(&ws.err, sizeof(unsigned));
  ws.nodes_cap = (int)ntab;
  if (e == cudaSuccess) e = cudaMemset(ws.err, 0, sizeof(unsigned));
  if (e == cudaSuccess) {
    // RoPE angles p * theta^(-2j/hd) in double precision, stored as fp32 cos/sin.
    std::vector<float2> tab((size_t)ws.tp_max * (dm.hd / 2));
    for (int p = 0; p < ws.tp_max; ++p)
      for (int j = 0; j < dm.hd / 2; ++j) {
        const double ang = (double)p * pow((double)dm.theta, -2.0 * j / dm.hd);
        tab[(size_t)j * ws.tp_max + p] = make_float2((float)cos(ang), (float)sin(ang));
      }
    e = cudaMemcpy(ws.rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice);
  }
  if (e == cudaSuccess) e = setup_memory_kernels(dm);
  if (e == cudaSuccess && dm.bf16) e = setup_tc_gemm();
  if (e == cudaSuccess && dm.bf16 && attention_tc_supported(dm)) e = setup_attention_tc();
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&ctx->capture_stream, cudaStreamNonBlocking);
  if (e != cudaSuccess) {
    armt_status s = cuda_fail(nullptr, e, "create");
    free_workspace(ctx->ws);
    if (ctx->capture_stream) cudaStreamDestroy(ctx->capture_stream);
    delete ctx;
    return s;
  }
  *out = ctx;
  return ARMT_OK;
}

extern "C" armt_status armt_destroy(armt_ctx* ctx) {
  if (!ctx) return ARMT_OK;
  if (ctx->graph_exec) cudaGraphExecDestroy(ctx->graph_exec);
  if (ctx->host_graph_exec) cudaGraphExecDestroy(ctx->host_graph_exec);
  if (ctx->capture_stream) cudaStreamDestroy(ctx->capture_stream);
  if (ctx->copy_in_stream) cudaStreamDestroy(ctx->copy_in_stream);
  if (ctx->copy_out_stream) cudaStreamDestroy(ctx->copy_out_stream);
  if (ctx->ov_stream) cudaStreamDestroy(ctx->ov_stream);
  for (cudaEvent_t ev : ctx->ov_ev)
    if (ev) cudaEventDestroy(ev);
  for (cudaEvent_t ev : ctx->host_events) cudaEventDestroy(ev);
  free_weights(ctx->w);
  free_workspace(ctx->ws);
  dfree(ctx->st_emb); dfree(ctx->st_out); dfree(ctx->st_A); dfree(ctx->st_z);
  delete ctx;
  return ARMT_OK;
}

extern "C" armt_status armt_set_schedule(armt_ctx* ctx, armt_schedule s) {
  if (!ctx) return ARMT_ERR_INVALID_ARG;
  if (s != ARMT_SCHED_DIAGONAL && s != ARMT_SCHED_SEQUENTIAL) return fail(ctx, ARMT_ERR_INVALID_ARG, "schedule");
  ctx->cfg.schedule = s;
  return ARMT_OK;
}

extern "C" armt_status armt_set_graph(armt_ctx* ctx, int enable) {
  if (!ctx) return ARMT_ERR_INVALID_ARG;
  ctx->use_graph = enable != 0;
  return ARMT_OK;
}

extern "C" armt_status armt_load_weights(armt_ctx* ctx, const armt_weights* wt) {
  if (!ctx) return ARMT_ERR_INVALID_ARG;
  const bool mem = ctx->dm.M > 0;   // the memory weights are read only with memory tokens
  if (!wt || !wt->attn_norm || !wt->mlp_norm || !wt->wq || !wt->wk || !wt->wv || !wt->wo || !wt->w_gate ||
      !wt->w_up || !wt->w_down ||
      (mem && (!wt->mem_emb || !wt->wq_mem || !wt->wk_mem || !wt->wv_mem || (ctx->dm.write_gate && !wt->w_beta))))
    return fail(ctx, ARMT_ERR_INVALID_ARG, "null weight pointer");
  const Dims& dm = ctx->dm;
  free_weights(ctx->w);
  Weights& w = ctx->w;
  const size_t as = act_size(dm);
  const int L = dm.L, d = dm.d, F = dm.F, Hh = dm.H * dm.hd, KVh = dm.KV * dm.hd;
  cudaError_t e = cudaSuccess;
  auto A = [&](auto** p, size_t bytes) { if (e == cudaSuccess) e = dalloc(p, bytes); };
  A(&w.mem_emb, (size_t)dm.M * d * 4);
  A(&w.w_qkv, (size_t)L * dm.nqkv * d * as);
  A(&w.w_o, (size_t)L * d * Hh * as);
  const int f_pad = dm.bf16 ? (F + 127) / 128 * 128 : F;
  A(&w.w_gu, (size_t)L * 2 * f_pad * d * as);
  A(&w.w_down, (size_t)L * d * F * as);
  const int ldkv = kv_ld(dm);
  if (mem) {
    A(&w.w_qm, (size_t)L * dm.dk * d * as);
    A(&w.w_kvm, (size_t)L * ldkv * d * as);
  }
  // staging for one layer's largest block (fp32)
  const size_t blk = std::max({(size_t)dm.nqkv * d, (size_t)d * Hh, 2 * (size_t)f_pad * d, (size_t)d * F,
                               (size_t)ldkv * d});
  float* stage = nullptr;
  A(&stage, blk * 4);
  if (e != cudaSuccess) {
    dfree(stage);
    free_weights(ctx->w);
    return cuda_fail(ctx, e, "allocate weights");
  }
  std::vector<float> host(blk);
  cudaStream_t st = 0;
  // folded: the block holds products W diag(g) (bf16 mode: of the bf16-rounded
  // W and g, exact in fp32), stored at fp16 precision; others are bf16 values
  auto put = [&](void* dst_base, size_t layer_elems, int l, size_t n_elems, bool folded = false) {
    if (e != cudaSuccess) return;
    e = cudaMemcpy(stage, host.data(), n_elems * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
      e = launch_convert(stage, (char*)dst_base + (size_t)l * layer_elems * as, n_elems,
                         dm.bf16 ? (folded ? CONVERT_F16 : CONVERT_BF16_AS_F16) : CONVERT_COPY_F32, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  };
  // bf16 round to nearest even of an fp32 value (host); identity in fp32 mode
  auto to_model = [&](float x) {
    if (!dm.bf16) return x;
    uint32_t b;
    memcpy(&b, &x, 4);
    b = (b + 0x7FFFu + ((b >> 16) & 1u)) & 0xFFFF0000u;
    memcpy(&x, &b, 4);
    return x;
  };
  // rows of W scaled by the RMSNorm gain on the input dimension: (x*g) W^T = x (W diag g)^T.
  // bf16 mode: the product of the bf16-rounded W and g (16 significant bits,
  // exact in fp32) is stored as fp16, 3 bits finer than rounding it to bf16.
  auto scaled_rows = [&](float* dst, const float* src, int rows, const float* gain) {
    for (int r = 0; r < rows; ++r)
      for (int k = 0; k < d; ++k) dst[(size_t)r * d + k] = to_model(src[(size_t)r * d + k]) * to_model(gain[k]);
  };
  for (int l = 0; l < L && e == cudaSuccess; ++l) {
    const float* ga = wt->attn_norm + (size_t)l * d;
    const float* gm = wt->mlp_norm + (size_t)l * d;
    scaled_rows(host.data(), wt->wq + (size_t)l * Hh * d, Hh, ga);
    scaled_rows(host.data() + (size_t)Hh * d, wt->wk + (size_t)l * KVh * d, KVh, ga);
    scaled_rows(host.data() + (size_t)(Hh + KVh) * d, wt->wv + (size_t)l * KVh * d, KVh, ga);
    put(w.w_qkv, (size_t)dm.nqkv * d, l, (size_t)dm.nqkv * d, true);
    memcpy(host.data(), wt->wo + (size_t)l * d * Hh, (size_t)d * Hh * 4);
    put(w.w_o, (size_t)d * Hh, l, (size_t)d * Hh);
    if (dm.bf16) {
      // tensor-core layout: blocks of 128 gate rows followed by the matching
      // 128 up rows, so one 256-column tile holds both halves of SwiGLU;
      // rows past F are zero
      std::fill(host.begin(), host.begin() + 2 * (size_t)f_pad * d, 0.f);
      for (int b = 0; b < f_pad / 128; ++b) {
        const int rows = std::min(128, F - b * 128);
        if (rows <= 0) break;
        scaled_rows(host.data() + (size_t)(2 * b) * 128 * d, wt->w_gate + ((size_t)l * F + b * 128) * d, rows, gm);
        scaled_rows(host.data() + (size_t)(2 * b + 1) * 128 * d, wt->w_up + ((size_t)l * F + b * 128) * d, rows, gm);
      }
    } else {
      scaled_rows(host.data(), wt->w_gate + (size_t)l * F * d, F, gm);
      scaled_rows(host.data() + (size_t)F * d, wt->w_up + (size_t)l * F * d, F, gm);
    }
    put(w.w_gu, 2 * (size_t)f_pad * d, l, 2 * (size_t)f_pad * d, true);
    memcpy(host.data(), wt->w_down + (size_t)l * d * F, (size_t)d * F * 4);
    put(w.w_down, (size_t)d * F, l, (size_t)d * F);
    if (!mem) continue;
    memcpy(host.data(), wt->wq_mem + (size_t)l * dm.dk * d, (size_t)dm.dk * d * 4);
    put(w.w_qm, (size_t)dm.dk * d, l, (size_t)dm.dk * d);
    // [Wk_mem; Wv_mem; w_beta; zero rows] (the gate row and its padding only for the gated write)
    memcpy(host.data(), wt->wk_mem + (size_t)l * dm.dk * d, (size_t)dm.dk * d * 4);
    memcpy(host.data() + (size_t)dm.dk * d, wt->wv_mem + (size_t)l * d * d, (size_t)d * d * 4);
    if (dm.write_gate) {
      std::fill(host.begin() + (size_t)(dm.dk + d) * d, host.begin() + (size_t)ldkv * d, 0.f);
      memcpy(host.data() + (size_t)(dm.dk + d) * d, wt->w_beta + (size_t)l * d, (size_t)d * 4);
    }
    put(w.w_kvm, (size_t)ldkv * d, l, (size_t)ldkv * d);
  }
  if (e == cudaSuccess && mem) e = cudaMemcpy(w.mem_emb, wt->mem_emb, (size_t)dm.M * d * 4, cudaMemcpyHostToDevice);
  dfree(stage);
  if (e != cudaSuccess) {
    free_weights(ctx->w);
    return cuda_fail(ctx, e, "upload weights");
  }
  w.loaded = true;
  return ARMT_OK;
}

extern "C" armt_status armt_forward(armt_ctx* ctx, const void* emb, int S, int seg_len, void* out_hidden,
                                    float* out_A, float* out_z, void* stream) {
  armt_status s = check_forward_args(ctx, emb, S, seg_len, out_hidden, out_A, out_z);
  if (s != ARMT_OK) return s;
  return forward_impl(ctx, emb, S, seg_len, out_hidden, out_A, out_z, (cudaStream_t)stream);
}

extern "C" armt_status armt_forward_ex(armt_ctx* ctx, const void* emb, int S, int seg_len, void* out_hidden,
                                       float* A, float* z, int carry_state, void* stream) {
  armt_status s = check_forward_args(ctx, emb, S, seg_len, out_hidden, A, z);
  if (s != ARMT_OK) return s;
  if (carry_state != 0 && carry_state != 1) return fail(ctx, ARMT_ERR_INVALID_ARG, "carry_state must be 0 or 1");
  return forward_impl(ctx, emb, S, seg_len, out_hidden, A, z, (cudaStream_t)stream, carry_state == 1);
}

extern "C" armt_status armt_stage_wave(armt_ctx* ctx, int S, int seg_len, int wave, int layer_offset,
                                       int total_layers, const void* emb, const float* in_rows, float* out_rows,
                                       void* out_hidden, float* A, float* z, int carry_state, void* stream) {
  if (!ctx) return ARMT_ERR_INVALID_ARG;
  if (!A || !z) return fail(ctx, ARMT_ERR_INVALID_ARG, "null state buffer");
  if (S < 1 || seg_len < 1) return fail(ctx, ARMT_ERR_INVALID_ARG, "S and seg_len must be >= 1");
  if (carry_state != 0 && carry_state != 1) return fail(ctx, ARMT_ERR_INVALID_ARG, "carry_state must be 0 or 1");
  if (!ctx->w.loaded) return fail(ctx, ARMT_ERR_NOT_LOADED, "weights not loaded");
  if (S > ctx->cfg.max_segments) return fail(ctx, ARMT_ERR_SHAPE, "S > max_segments");
  if (seg_len > ctx->cfg.max_seg_len) return fail(ctx, ARMT_ERR_SHAPE, "seg_len > max_seg_len");
  const int nl = ctx->dm.L;
  if (layer_offset < 0 || total_layers < 1 || layer_offset + nl > total_layers)
    return fail(ctx, ARMT_ERR_INVALID_ARG, "layer block outside the model");
  if (wave < 0 || wave >= S + total_layers - 1) return fail(ctx, ARMT_ERR_INVALID_ARG, "wave out of range");
  const int first = layer_offset, last = layer_offset + nl - 1;
  const bool has_first = wave - first >= 0 && wave - first < S;
  const bool has_last = wave - last >= 0 && wave - last < S;
  const bool final_stage = last == total_layers - 1;
  if (has_first && first == 0 && !emb) return fail(ctx, ARMT_ERR_INVALID_ARG, "null emb");
  if (has_first && first > 0 && !in_rows) return fail(ctx, ARMT_ERR_INVALID_ARG, "null in_rows");
  if (has_last && !final_stage && !out_rows) return fail(ctx, ARMT_ERR_INVALID_ARG, "null out_rows");
  if (has_last && final_stage && !out_hidden) return fail(ctx, ARMT_ERR_INVALID_ARG, "null out_hidden");
  cudaStream_t st = (cudaStream_t)stream;
  if (ctx->stage_S != S || ctx->stage_offset != layer_offset || ctx->stage_total != total_layers) {
    std::vector<NodeEntry> tab;
    build_stage_table(S, nl, layer_offset, total_layers, ctx->ws.slots, tab, ctx->stage_waves);
    if ((int)tab.size() > ctx->ws.nodes_cap) return fail(ctx, ARMT_ERR_SHAPE, "node table too large");
    // stream-ordered after the work that may still read the previous table
    ARMT_TRY(cudaMemcpyAsync(ctx->ws.nodes, tab.data(), tab.size() * sizeof(NodeEntry), cudaMemcpyHostToDevice, st),
             "upload stage table");
    ARMT_TRY(cudaStreamSynchronize(st), "upload stage table");
    ctx->table_S = -1;   // the forward's table is gone
    ctx->stage_S = S;
    ctx->stage_offset = layer_offset;
    ctx->stage_total = total_layers;
  }
  const Dims& dm = ctx->dm;
  if (wave == 0 && !carry_state) {
    ARMT_TRY(cudaMemsetAsync(A, 0, (size_t)dm.L * dm.d * dm.P * sizeof(float), st), "zero A");
    ARMT_TRY(cudaMemsetAsync(z, 0, (size_t)dm.L * dm.P * sizeof(float), st), "zero z");
  }
  const Wave& wv = ctx->stage_waves[wave];
  if (wv.count == 0) return ARMT_OK;
  Launcher L;
  const float* sin = first > 0 ? in_rows : nullptr;
  float* sout = final_stage ? nullptr : out_rows;
  void* out = final_stage ? out_hidden : nullptr;
  if (dm.bf16) enqueue_wave_tc(ctx, wv, seg_len, emb, out, A, z, st, L, nullptr, sin, sout);
  else enqueue_wave(ctx, wv, seg_len, emb, out, A, z, st, L, sin, sout);
  if (L.err != cudaSuccess) return cuda_fail(ctx, L.err, L.where);
  return ARMT_OK;
}

namespace {

bool host_page_locked(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

// Host-buffer forward on page-locked buffers as one graph over three streams:
// the embeddings of segment s are copied in on one stream and the wave that
// starts segment s (its layer-0 node) waits for that copy only; the hidden
// rows of segment s are copied out on another stream as soon as the wave
// holding its last-layer node has run; A and z follow the last wave.  The
// copies thus overlap the forward instead of bracketing it.
armt_status forward_host_overlapped(armt_ctx* ctx, const void* emb_host, int S, int T, void* out_host,
                                    float* A_host, float* z_host, cudaStream_t st) {
  const Dims& dm = ctx->dm;
  armt_status s = ensure_table(ctx, S, st);
  if (s != ARMT_OK) return s;
  armt_ctx::GraphKey key;
  key.S = S; key.T = T; key.sched = (int)ctx->cfg.schedule;
  key.emb = emb_host; key.out = out_host; key.A = A_host; key.z = z_host;
  const armt_ctx::GraphKey& k0 = ctx->host_key;
  const bool same = ctx->host_graph_exec && k0.S == key.S && k0.T == key.T && k0.sched == key.sched &&
                    k0.emb == key.emb && k0.out == key.out && k0.A == key.A && k0.z == key.z;
  if (!same) {
    if (ctx->host_graph_exec) {
      cudaGraphExecDestroy(ctx->host_graph_exec);
      ctx->host_graph_exec = nullptr;
    }
    if (!ctx->copy_in_stream) ARMT_TRY(cudaStreamCreateWithFlags(&ctx->copy_in_stream, cudaStreamNonBlocking), "copy stream");
    if (!ctx->copy_out_stream) ARMT_TRY(cudaStreamCreateWithFlags(&ctx->copy_out_stream, cudaStreamNonBlocking), "copy stream");
    const size_t need = 2 * (size_t)S + 3;
    while (ctx->host_events.size() < need) {
      cudaEvent_t ev;
      ARMT_TRY(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming), "event");
      ctx->host_events.push_back(ev);
    }
    cudaEvent_t* ev_in = ctx->host_events.data();        // [S]
    cudaEvent_t* ev_out = ev_in + S;                      // [S]
    cudaEvent_t ev_fork = ev_out[S], ev_join_in = ev_out[S + 1], ev_join_out = ev_out[S + 2];
    cudaStream_t s1 = ctx->capture_stream, s2 = ctx->copy_in_stream, s3 = ctx->copy_out_stream;
    const size_t as = act_size(dm);
    const size_t seg_bytes = (size_t)T * dm.d * as;
    ARMT_TRY(cudaStreamBeginCapture(s1, cudaStreamCaptureModeThreadLocal), "begin capture");
    cudaError_t e = cudaSuccess;
    const char* where = "host forward capture";
    auto C = [&](cudaError_t r, const char* w) { if (e == cudaSuccess && r != cudaSuccess) { e = r; where = w; } };
    C(cudaEventRecord(ev_fork, s1), "fork");
    C(cudaStreamWaitEvent(s2, ev_fork, 0), "fork");
    C(cudaStreamWaitEvent(s3, ev_fork, 0), "fork");
    for (int sg = 0; sg < S && e == cudaSuccess; ++sg) {
      C(cudaMemcpyAsync((char*)ctx->st_emb + sg * seg_bytes, (const char*)emb_host + sg * seg_bytes, seg_bytes,
                        cudaMemcpyHostToDevice, s2), "copy emb in");
      C(cudaEventRecord(ev_in[sg], s2), "copy emb in");
    }
    C(cudaMemsetAsync(ctx->st_A, 0, (size_t)dm.L * dm.d * dm.P * sizeof(float), s1), "zero A");
    C(cudaMemsetAsync(ctx->st_z, 0, (size_t)dm.L * dm.P * sizeof(float), s1), "zero z");
    Launcher L;
    WriteOverlap* ov = (ctx->overlap_write && dm.bf16 && dm.M > 0) ? write_overlap(ctx) : nullptr;
    for (const Wave& wv : ctx->waves) {
      if (e != cudaSuccess) break;
      if (wv.first_layer_seg >= 0) C(cudaStreamWaitEvent(s1, ev_in[wv.first_layer_seg], 0), "wait emb");
      if (dm.bf16) enqueue_wave_tc(ctx, wv, T, ctx->st_emb, ctx->st_out, ctx->st_A, ctx->st_z, s1, L, ov);
      else enqueue_wave(ctx, wv, T, ctx->st_emb, ctx->st_out, ctx->st_A, ctx->st_z, s1, L);
      C(L.err, L.where);
      if (wv.last_layer_seg >= 0) {
        const int sg = wv.last_layer_seg;
        C(cudaEventRecord(ev_out[sg], s1), "segment done");
        C(cudaStreamWaitEvent(s3, ev_out[sg], 0), "segment done");
        C(cudaMemcpyAsync((char*)out_host + sg * seg_bytes, (const char*)ctx->st_out + sg * seg_bytes, seg_bytes,
                          cudaMemcpyDeviceToHost, s3), "copy out");
      }
    }
    C(join_write(ov, s1), "join the memory write");
    C(cudaMemcpyAsync(A_host, ctx->st_A, (size_t)dm.L * dm.d * dm.P * 4, cudaMemcpyDeviceToHost, s1), "copy A");
    C(cudaMemcpyAsync(z_host, ctx->st_z, (size_t)dm.L * dm.P * 4, cudaMemcpyDeviceToHost, s1), "copy z");
    C(cudaEventRecord(ev_join_in, s2), "join");
    C(cudaStreamWaitEvent(s1, ev_join_in, 0), "join");
    C(cudaEventRecord(ev_join_out, s3), "join");
    C(cudaStreamWaitEvent(s1, ev_join_out, 0), "join");
    cudaGraph_t graph = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(s1, &graph);
    if (e == cudaSuccess) e = ce;
    if (e == cudaSuccess) e = cudaGraphInstantiate(&ctx->host_graph_exec, graph, 0);
    if (graph) cudaGraphDestroy(graph);
    if (e != cudaSuccess) {
      ctx->host_graph_exec = nullptr;
      return cuda_fail(ctx, e, where);
    }
    ctx->host_key = key;
  }
  ARMT_TRY(cudaGraphLaunch(ctx->host_graph_exec, st), "graph launch");
  ARMT_TRY(cudaStreamSynchronize(st), "host forward sync");
  return ARMT_OK;
}

}  // namespace

extern "C" armt_status armt_forward_host(armt_ctx* ctx, const void* emb_host, int S, int seg_len,
                                         void* out_hidden_host, float* out_A_host, float* out_z_host,
                                         void* stream) {
  armt_status s = check_forward_args(ctx, emb_host, S, seg_len, out_hidden_host, out_A_host, out_z_host);
  if (s != ARMT_OK) return s;
  const Dims& dm = ctx->dm;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t max_tok = (size_t)ctx->cfg.max_segments * ctx->cfg.max_seg_len;
  const size_t as = act_size(dm);
  if (!ctx->st_emb) {
    cudaError_t e = dalloc(&ctx->st_emb, max_tok * dm.d * as);
    if (e == cudaSuccess) e = dalloc(&ctx->st_out, max_tok * dm.d * as);
    if (e == cudaSuccess) e = dalloc(&ctx->st_A, (size_t)dm.L * dm.d * dm.P * 4);
    if (e == cudaSuccess) e = dalloc(&ctx->st_z, (size_t)dm.L * dm.P * 4);
    if (e != cudaSuccess) {
      dfree(ctx->st_emb); dfree(ctx->st_out); dfree(ctx->st_A); dfree(ctx->st_z);
      ctx->st_emb = ctx->st_out = nullptr; ctx->st_A = ctx->st_z = nullptr;
      return cuda_fail(ctx, e, "allocate host-forward staging");
    }
  }
  const size_t tok = (size_t)S * seg_len;
  if (ctx->use_graph && host_page_locked(emb_host) && host_page_locked(out_hidden_host) &&
      host_page_locked(out_A_host) && host_page_locked(out_z_host))
    return forward_host_overlapped(ctx, emb_host, S, seg_len, out_hidden_host, out_A_host, out_z_host, st);
  ARMT_TRY(cudaMemcpyAsync(ctx->st_emb, emb_host, tok * dm.d * as, cudaMemcpyHostToDevice, st), "copy emb in");
  s = forward_impl(ctx, ctx->st_emb, S, seg_len, ctx->st_out, ctx->st_A, ctx->st_z, st);
  if (s != ARMT_OK) return s;
  ARMT_TRY(cudaMemcpyAsync(out_hidden_host, ctx->st_out, tok * dm.d * as, cudaMemcpyDeviceToHost, st), "copy out");
  ARMT_TRY(cudaMemcpyAsync(out_A_host, ctx->st_A, (size_t)dm.L * dm.d * dm.P * 4, cudaMemcpyDeviceToHost, st), "copy A");
  ARMT_TRY(cudaMemcpyAsync(out_z_host, ctx->st_z, (size_t)dm.L * dm.P * 4, cudaMemcpyDeviceToHost, st), "copy z");
  ARMT_TRY(cudaStreamSynchronize(st), "host forward sync");
  return ARMT_OK;
}

extern "C" armt_status armt_device_status(armt_ctx* ctx, void* stream) {
  if (!ctx) return ARMT_ERR_INVALID_ARG;
  ARMT_TRY(cudaStreamSynchronize((cudaStream_t)stream), "stream");
  unsigned flag = 0;
  ARMT_TRY(cudaMemcpy(&flag, ctx->ws.err, sizeof(unsigned), cudaMemcpyDeviceToHost), "read error word");
  if (flag) {
    ARMT_TRY(cudaMemset(ctx->ws.err, 0, sizeof(unsigned)), "clear error word");
    return fail(ctx, ARMT_ERR_DEVICE_TIMEOUT, "a kernel's bounded wait timed out");
  }
  return ARMT_OK;
}

extern "C" int armt_kernel_kinds(void) { return N_KINDS; }

extern "C" const char* armt_kernel_kind_name(int k) { return (k >= 0 && k < N_KINDS) ? KIND_NAMES[k] : nullptr; }

extern "C" armt_status armt_profile_forward(armt_ctx* ctx, const void* emb, int S, int seg_len, void* out_hidden,
                                            float* out_A, float* out_z, void* stream, double* ms, int* launches) {
  armt_status s = check_forward_args(ctx, emb, S, seg_len, out_hidden, out_A, out_z);
  if (s != ARMT_OK) return s;
  if (!ms || !launches) return fail(ctx, ARMT_ERR_INVALID_ARG, "null profile arrays");
  cudaStream_t st = (cudaStream_t)stream;
  s = ensure_table(ctx, S, st);
  if (s != ARMT_OK) return s;
  Launcher L;
  L.profile = true;
  L.pstream = st;
  L.ev.reserve(2 * 64 * ctx->waves.size());
  s = enqueue_forward(ctx, emb, S, seg_len, out_hidden, out_A, out_z, st, L);
  if (s != ARMT_OK) return s;
  ARMT_TRY(cudaStreamSynchronize(st), "profile sync");
  for (size_t i = 0; i < L.kinds.size(); ++i) {
    float t = 0.f;
    ARMT_TRY(cudaEventElapsedTime(&t, L.ev[2 * i], L.ev[2 * i + 1]), "event elapsed");
    const int k = L.kinds[i];
    if (k >= 0) {
      ms[k] += t;
      launches[k] += 1;
    }
  }
  return ARMT_OK;
}

extern "C" armt_status armt_launch_count(armt_ctx* ctx, int S, int* out_count) {
  if (!ctx || !out_count || S < 1) return ARMT_ERR_INVALID_ARG;
  if (S > ctx->cfg.max_segments) return fail(ctx, ARMT_ERR_SHAPE, "S > max_segments");
  std::vector<NodeEntry> tab;
  std::vector<Wave> waves;
  build_table(S, ctx->dm.L, ctx->ws.slots, ctx->cfg.schedule, tab, waves);
  std::vector<Wave> saved;
  saved.swap(ctx->waves);
  ctx->waves = waves;
  Launcher L;
  L.dry = true;
  enqueue_forward(ctx, nullptr, S, ctx->cfg.max_seg_len, nullptr, nullptr, nullptr, 0, L);
  ctx->waves.swap(saved);
  *out_count = L.count;
  return ARMT_OK;
}
