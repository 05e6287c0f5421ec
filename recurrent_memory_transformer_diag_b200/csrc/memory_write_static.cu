// Delta-rule memory write that allocates no device memory.
//
// armt_memory_write takes its scratch (projected keys/values, DPFP features,
// Gram matrix, per-row scalars) from cudaMallocAsync on every call.  Some
// callers cannot allocate at call time: a host framework that has reserved
// the device memory for its own allocator, a real-time loop whose memory
// budget is fixed at start-up, or a plug-in whose host application forbids
// device allocation after initialisation.  This variant runs the same kernels
// with its scratch in a fixed array of the library's device image instead.
//
// The array is a file-scope __device__ variable: every device that loads the
// library holds it (1 MiB) until the process exits, and every call shares it.
// Host code cannot use the array's name as a device address (on the host it
// is only a stand-in symbol); the device address is looked up once per device
// with cudaGetSymbolAddress and cached.
#include <mutex>

#include "armt_internal.cuh"

using namespace armt;

namespace {

// 256 Ki floats = 1 MiB of scratch per device.
constexpr size_t STATIC_SCRATCH_FLOATS = 256 * 1024;
static __device__ __align__(256) float g_write_scratch[STATIC_SCRATCH_FLOATS];

constexpr int MAX_DEVICES = 64;
std::mutex g_scratch_mu;
float* g_scratch_dev[MAX_DEVICES] = {};

// Device address of g_write_scratch on the current device (looked up once per
// device, with that device current).
cudaError_t scratch_on_current_device(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_dev[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_write_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_dev[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_dev[dev];
  return cudaSuccess;
}

// Every sub-buffer starts on a 16-byte boundary (a multiple of 4 floats):
// the update kernel reads the DPFP features as float4.
size_t pad4(size_t n) { return (n + 3) & ~(size_t)3; }

// Floats of scratch one call needs: node entry (4), projected [k | v] rows,
// DPFP features, Gram matrix, coefficients and gammas, each padded to 4.
size_t scratch_floats(int M, int d, int d_key, int P) {
  return 4 + pad4((size_t)M * (d_key + d)) + pad4((size_t)M * P) + pad4((size_t)M * M) + pad4(M) + pad4(M);
}

armt_status to_status(cudaError_t e) {
  if (e == cudaSuccess) return ARMT_OK;
  cudaGetLastError();
  return ARMT_ERR_CUDA;
}

}  // namespace

extern "C" armt_status armt_memory_write_static(int M, int d, int d_key, int nu, float eps, const float* m,
                                                const float* wk, const float* wv, float* A, float* z,
                                                void* stream) {
  if (M < 1 || d < 1 || d_key < 1 || nu < 1 || !(eps > 0.f) || !m || !wk || !wv || !A || !z)
    return ARMT_ERR_INVALID_ARG;
  if (M > 32 || nu > 2 * d_key || 2 * d_key * nu > 1024) return ARMT_ERR_UNSUPPORTED;
  Dims dm{};
  dm.L = 1; dm.d = d; dm.M = M; dm.dk = d_key; dm.nu = nu; dm.P = 2 * d_key * nu; dm.mem_eps = eps;
  dm.bf16 = false;
  if (((size_t)dm.M * dm.P + (size_t)dm.M * dm.M + 17 * dm.M) * 4 > 200 * 1024 || memw_phi_smem(dm) > 200 * 1024)
    return ARMT_ERR_UNSUPPORTED;
  if (scratch_floats(M, d, d_key, dm.P) > STATIC_SCRATCH_FLOATS) return ARMT_ERR_SHAPE;
  float* scratch = nullptr;
  cudaError_t e = scratch_on_current_device(&scratch);
  if (e != cudaSuccess) return to_status(e);
  e = setup_memory_kernels(dm);
  if (e != cudaSuccess) return to_status(e);
  cudaStream_t st = (cudaStream_t)stream;
  NodeEntry* node = reinterpret_cast<NodeEntry*>(scratch);   // (segment 0, layer 0, slot 0)
  float* kv = scratch + 4;
  float* phik = kv + pad4((size_t)M * (d_key + d));
  float* gram = phik + pad4((size_t)M * dm.P);
  float* coef = gram + pad4((size_t)M * M);
  float* gamma = coef + pad4(M);
  // The array keeps the previous call's contents: the node entry must read as
  // zeros; everything else is fully written below before it is read.
  e = cudaMemsetAsync(node, 0, sizeof(NodeEntry), st);
  if (e == cudaSuccess) {   // k = m Wk^T into columns [0, d_key) of the [M][d_key + d] rows
    GemmArgs g{};
    g.nodes = node; g.n_nodes = 1; g.M = M; g.N = d_key; g.K = d;
    g.A = m; g.lda = d; g.B = wk; g.ldb = d;
    g.C = kv; g.ldc = d_key + d;
    g.epi = EPI_STORE_F32;
    e = launch_simt_gemm(g, st);
  }
  if (e == cudaSuccess) {   // v = m Wv^T into columns [d_key, d_key + d)
    GemmArgs g{};
    g.nodes = node; g.n_nodes = 1; g.M = M; g.N = d; g.K = d;
    g.A = m; g.lda = d; g.B = wv; g.ldb = d;
    g.C = kv + d_key; g.ldc = d_key + d;
    g.epi = EPI_STORE_F32;
    e = launch_simt_gemm(g, st);
  }
  if (e == cudaSuccess) e = launch_memw_phi(dm, node, 1, kv, z, phik, gram, coef, gamma, nullptr, st);
  if (e == cudaSuccess) e = launch_memw_update(dm, node, 1, kv, phik, gram, coef, nullptr, A, st);
  return to_status(e);
}
