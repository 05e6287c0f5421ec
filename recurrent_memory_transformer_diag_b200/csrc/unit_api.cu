// Unit entry points: one grouped kernel at a time on caller buffers, so each
// kernel can be checked against the oracle on its own.
#include <vector>

#include "armt_internal.cuh"

using namespace armt;

namespace {

armt_status to_status(cudaError_t e) {
  if (e == cudaSuccess) return ARMT_OK;
  cudaGetLastError();
  return e == cudaErrorMemoryAllocation ? ARMT_ERR_OOM : ARMT_ERR_CUDA;
}

}  // namespace

#include "tc_gemm.cuh"

extern "C" armt_status armt_grouped_gemm(armt_dtype dtype, int G, int m, int n, int k, const void* A,
                                         const void* B, int num_b, const int* bidx, float* C, void* stream) {
  if (G < 1 || m < 1 || n < 1 || k < 1 || num_b < 1 || !A || !B || !bidx || !C) return ARMT_ERR_INVALID_ARG;
  if (dtype != ARMT_FP32 && dtype != ARMT_BF16 && dtype != ARMT_F16 && dtype != ARMT_TF32)
    return ARMT_ERR_INVALID_ARG;
  std::vector<NodeEntry> tab(G);
  for (int g = 0; g < G; ++g) {
    if (bidx[g] < 0 || bidx[g] >= num_b) return ARMT_ERR_INVALID_ARG;
    tab[g] = make_int4(g, bidx[g], g, 0);
  }
  if (dtype != ARMT_FP32 && !tc_gemm_supported(m, n, k)) return ARMT_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  NodeEntry* dnodes = nullptr;
  cudaError_t e = cudaMallocAsync((void**)&dnodes, G * sizeof(NodeEntry) + 16, st);
  if (e != cudaSuccess) return to_status(e);
  unsigned* derr = reinterpret_cast<unsigned*>(dnodes + G);
  unsigned herr = 0;
  e = cudaMemcpyAsync(dnodes, tab.data(), G * sizeof(NodeEntry), cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(derr, 0, sizeof(unsigned), st);
  if (e == cudaSuccess) {
    if (dtype != ARMT_FP32) {
      e = launch_tc_gemm_unit(G, m, n, k, A, B, num_b, dnodes, C, derr,
                              dtype == ARMT_BF16 ? 1 : (dtype == ARMT_TF32 ? 2 : 0), st);
    } else {
      GemmArgs g{};
      g.nodes = dnodes; g.n_nodes = G; g.M = m; g.N = n; g.K = k;
      g.A = A; g.a_slot_stride = (long long)m * k; g.lda = k;
      g.B = B; g.b_layer_stride = (long long)n * k; g.ldb = k;
      g.C = C; g.c_slot_stride = (long long)m * n; g.ldc = n;
      g.epi = EPI_STORE_F32;
      e = launch_simt_gemm(g, st);
    }
  }
  if (e == cudaSuccess) e = cudaMemcpyAsync(&herr, derr, sizeof(unsigned), cudaMemcpyDeviceToHost, st);
  cudaError_t e2 = cudaStreamSynchronize(st);   // the host table must outlive the copy
  cudaFreeAsync(dnodes, st);
  if (e == cudaSuccess) e = e2;
  if (e == cudaSuccess && herr) return ARMT_ERR_DEVICE_TIMEOUT;
  return to_status(e);
}

extern "C" armt_status armt_memory_write(int M, int d, int d_key, int nu, float eps, const float* m,
                                         const float* wk, const float* wv, float* A, float* z, void* stream) {
  if (M < 1 || d < 1 || d_key < 1 || nu < 1 || !(eps > 0.f) || !m || !wk || !wv || !A || !z)
    return ARMT_ERR_INVALID_ARG;
  if (M > 32 || nu > 2 * d_key || 2 * d_key * nu > 1024) return ARMT_ERR_UNSUPPORTED;
  Dims dm{};
  dm.L = 1; dm.d = d; dm.M = M; dm.dk = d_key; dm.nu = nu; dm.P = 2 * d_key * nu; dm.mem_eps = eps;
  dm.bf16 = false;
  if (((size_t)dm.M * dm.P + (size_t)dm.M * dm.M + 17 * dm.M) * 4 > 200 * 1024 || memw_phi_smem(dm) > 200 * 1024)
    return ARMT_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = setup_memory_kernels(dm);
  if (e != cudaSuccess) return to_status(e);
  // sub-buffers padded to 4 floats: each starts on a 16-byte boundary (the
  // update kernel reads the DPFP features as float4)
  auto pad4 = [](size_t n) { return (n + 3) & ~(size_t)3; };
  const size_t n_w = pad4((size_t)(d_key + d) * d), n_kv = pad4((size_t)M * (d_key + d)),
               n_ph = pad4((size_t)M * dm.P), n_m = pad4(M);
  const size_t bytes = (n_w + n_kv + n_ph + 2 * n_m + (size_t)M * M) * sizeof(float) + sizeof(NodeEntry);
  char* scratch = nullptr;
  e = cudaMallocAsync((void**)&scratch, bytes, st);
  if (e != cudaSuccess) return to_status(e);
  NodeEntry* node = (NodeEntry*)scratch;
  float* w_kv = (float*)(scratch + sizeof(NodeEntry));
  float* kv = w_kv + n_w;
  float* phik = kv + n_kv;
  float* coef = phik + n_ph;
  float* gamma = coef + n_m;
  float* gram = gamma + n_m;
  static const NodeEntry one = {0, 0, 0, 0};
  e = cudaMemcpyAsync(node, &one, sizeof(NodeEntry), cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(w_kv, wk, (size_t)d_key * d * 4, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(w_kv + (size_t)d_key * d, wv, (size_t)d * d * 4, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) {
    GemmArgs g{};
    g.nodes = node; g.n_nodes = 1; g.M = M; g.N = d_key + d; g.K = d;
    g.A = m; g.a_slot_stride = 0; g.lda = d;
    g.B = w_kv; g.b_layer_stride = 0; g.ldb = d;
    g.C = kv; g.c_slot_stride = 0; g.ldc = d_key + d;
    g.epi = EPI_STORE_F32;
    e = launch_simt_gemm(g, st);
  }
  if (e == cudaSuccess) e = launch_memw_phi(dm, node, 1, kv, z, phik, gram, coef, gamma, nullptr, st);
  if (e == cudaSuccess) e = launch_memw_update(dm, node, 1, kv, phik, gram, coef, nullptr, A, st);
  cudaError_t e2 = cudaFreeAsync(scratch, st);
  if (e == cudaSuccess) e = e2;
  return to_status(e);
}

// The bounded-wait error path of the grouped GEMM, on demand: one 128 x 256
// tile with K = 1024 (16 k-blocks, more than the pipeline's stages) whose
// producer is told to issue no copies.  The MMA warp's wait for the first
// stage then runs out (about one second), it records the timeout in the
// error word and raises the CTA's abort flag, the producer and epilogue warps
// leave their waits, every warp reaches the final barrier and TMEM is freed.
extern "C" armt_status armt_test_bounded_wait(void* stream) {
  cudaStream_t st = (cudaStream_t)stream;
  const int m = 128, n = 256, k = 1024;
  const size_t bytes_a = (size_t)m * k * 2, bytes_b = (size_t)n * k * 2, bytes_c = (size_t)m * n * 4;
  char* buf = nullptr;
  cudaError_t e = cudaMallocAsync((void**)&buf, bytes_a + bytes_b + bytes_c + 256, st);
  if (e != cudaSuccess) return to_status(e);
  NodeEntry* dnode = reinterpret_cast<NodeEntry*>(buf + bytes_a + bytes_b + bytes_c);
  unsigned* derr = reinterpret_cast<unsigned*>(dnode + 1);
  unsigned herr = 0;
  static const NodeEntry one = {0, 0, 0, 0};
  e = cudaMemsetAsync(buf, 0, bytes_a + bytes_b, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dnode, &one, sizeof(NodeEntry), cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(derr, 0, sizeof(unsigned), st);
  if (e == cudaSuccess)
    e = launch_tc_gemm_unit(1, m, n, k, buf, buf + bytes_a, 1, dnode, reinterpret_cast<float*>(buf + bytes_a + bytes_b),
                            derr, 0, st, /*debug_no_loads=*/1);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&herr, derr, sizeof(unsigned), cudaMemcpyDeviceToHost, st);
  cudaError_t e2 = cudaStreamSynchronize(st);
  cudaFreeAsync(buf, st);
  if (e == cudaSuccess) e = e2;
  if (e != cudaSuccess) return to_status(e);
  return (herr & ERR_WAIT_TIMEOUT_MASK) ? ARMT_ERR_DEVICE_TIMEOUT : ARMT_OK;
}
