// ARMT associative-memory write (delta rule) for every node of a wave.
//
// The pages name ARMT as the layer-recurrent model Diagonal Batching targets
// (Pith review of arXiv 2506.05229, "The reading") and cite its DPFP feature
// map and delta-rule update (reference list, refs. 28, 29, 38) without
// printing them.  The reading implemented here, for node (s, l) with the M
// memory rows m_j of its layer output, k_j = Wk_mem m_j, v_j = Wv_mem m_j,
// phi_j = DPFP(k_j), and the state (A_l, z_l) left by segment s-1:
//   vbar_j  = A_l phi_j / (z_l . phi_j + eps)
//   gamma_j = clamp(1 - (z_l . phi_j) / (|phi_j|^2 + eps), 0, 1)
//   A_l    += sum_j (v_j - vbar_j) phi_j^T
//   z_l    += sum_j gamma_j phi_j
// with every j reading the state from before this write.
//
// Work split: memw_phi (one block per node) computes phi_j, the per-row
// scalars and the z update; memw_update streams A_l once, row by row: row i
// of the update needs only row i of the old A (vbar_j[i] = A[i,:] . phi_j),
// so each warp reads its row, forms the M dot products, applies the rank-M
// update and writes the row back -- one read and one write of A per node.
#include "armt_internal.cuh"

namespace armt {

__device__ __forceinline__ float warp_sum_m(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float block_sum(float v, float* sh) {
  v = warp_sum_m(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  float t = 0.f;
  const int nw = blockDim.x >> 5;
  for (int i = 0; i < nw; ++i) t += sh[i];
  return t;
}

// kv: [slot][M][dk + d] (k first), phik: [slot][M][P], coef/gamma: [slot][M]
__global__ void memw_phi_kernel(const NodeEntry* nodes, int M, int dk, int d, int P,
                                const float* kv, float* z_state, float* phik, float* coef,
                                float* gamma, float eps) {
  extern __shared__ float sh[];
  float* r = sh;                 // [2 dk]
  float* gam = r + 2 * dk;       // [M]
  float* red = gam + M;          // [32]
  const NodeEntry nd = nodes[blockIdx.x];
  const int slot = nd.z, layer = nd.y;
  float* z = z_state + (long long)layer * P;
  const int n2 = 2 * dk;
  for (int j = 0; j < M; ++j) {
    const float* k = kv + ((long long)slot * M + j) * (dk + d);
    __syncthreads();
    for (int c = threadIdx.x; c < dk; c += blockDim.x) {
      r[c] = fmaxf(k[c], 0.f);
      r[c + dk] = fmaxf(-k[c], 0.f);
    }
    __syncthreads();
    float* ph = phik + ((long long)slot * M + j) * P;
    float zp = 0.f, nn = 0.f;
    for (int p = threadIdx.x; p < P; p += blockDim.x) {
      const int n = p / n2 + 1, jj0 = p - (n - 1) * n2;
      int jj = (jj0 - n) % n2;
      if (jj < 0) jj += n2;
      const float f = r[jj0] * r[jj];
      ph[p] = f;
      zp = fmaf(z[p], f, zp);
      nn = fmaf(f, f, nn);
    }
    zp = block_sum(zp, red);
    nn = block_sum(nn, red);
    if (threadIdx.x == 0) {
      const float gm = fminf(fmaxf(1.f - zp / (nn + eps), 0.f), 1.f);
      gam[j] = gm;
      coef[(long long)slot * M + j] = 1.f / (zp + eps);
      gamma[(long long)slot * M + j] = gm;
    }
  }
  __syncthreads();   // every z . phi_j above read the old z; phi rows are visible block-wide
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < M; ++j) acc = fmaf(gam[j], phik[((long long)slot * M + j) * P + p], acc);
    z[p] += acc;
  }
}

cudaError_t launch_memw_phi(const Dims& dm, const NodeEntry* nodes, int n, const float* kv,
                            float* z_state, float* phik, float* coef, float* gamma, cudaStream_t st) {
  const size_t sh = (2 * dm.dk + dm.M + 32) * sizeof(float);
  memw_phi_kernel<<<n, 256, sh, st>>>(nodes, dm.M, dm.dk, dm.d, dm.P, kv, z_state, phik, coef, gamma,
                                      dm.mem_eps);
  return cudaGetLastError();
}

constexpr int MEMW_ROWS_PER_BLOCK = 64;

// A_state: [L][d][P] fp32 in place; a_act: optional bf16 copy [L][d][P].
// grid (ceil(d / ROWS_PER_BLOCK), nodes), 8 warps, one A row per warp per
// iteration; phi is staged once per block.
template <int MAXC>
__global__ void __launch_bounds__(256) memw_update_kernel(const NodeEntry* nodes, int M, int dk, int d, int P,
                                                          const float* kv, const float* phik,
                                                          const float* coef, float* A_state, bf16* a_act) {
  extern __shared__ float sh[];
  float* ph = sh;                    // [M][P]
  float* cf = ph + M * P;            // [M]
  float* delta = cf + M;             // [8][M]
  const NodeEntry nd = nodes[blockIdx.y];
  const int slot = nd.z, layer = nd.y;
  for (int e = threadIdx.x; e < M * P; e += blockDim.x) ph[e] = phik[(long long)slot * M * P + e];
  for (int e = threadIdx.x; e < M; e += blockDim.x) cf[e] = coef[(long long)slot * M + e];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i_end = min(d, (blockIdx.x + 1) * MEMW_ROWS_PER_BLOCK);
  for (int i = blockIdx.x * MEMW_ROWS_PER_BLOCK + warp; i < i_end; i += 8) {
    float* Arow = A_state + ((long long)layer * d + i) * P;
    float a[MAXC];
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int p = lane + 32 * c;
      a[c] = p < P ? Arow[p] : 0.f;
    }
    float* dl = delta + warp * M;
    for (int j = 0; j < M; ++j) {
      const float* pj = ph + j * P;
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < MAXC; ++c) {
        const int p = lane + 32 * c;
        if (p < P) dot = fmaf(a[c], pj[p], dot);
      }
      dot = warp_sum_m(dot);
      if (lane == 0) {
        const float v = kv[((long long)slot * M + j) * (dk + d) + dk + i];
        dl[j] = v - dot * cf[j];
      }
    }
    __syncwarp();
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int p = lane + 32 * c;
      if (p < P) {
        float acc = a[c];
        for (int j = 0; j < M; ++j) acc = fmaf(dl[j], ph[j * P + p], acc);
        Arow[p] = acc;
        if (a_act) a_act[((long long)layer * d + i) * P + p] = __float2bfloat16_rn(acc);
      }
    }
    __syncwarp();
  }
}

cudaError_t launch_memw_update(const Dims& dm, const NodeEntry* nodes, int n, const float* kv,
                               const float* phik, const float* coef, float* A_state, void* a_act,
                               cudaStream_t st) {
  dim3 grid((dm.d + MEMW_ROWS_PER_BLOCK - 1) / MEMW_ROWS_PER_BLOCK, n);
  const size_t sh = ((size_t)dm.M * dm.P + dm.M + 8 * dm.M) * sizeof(float);
  const int chunks = (dm.P + 31) / 32;
#define ARMT_MEMW_CASE(C)                                                                        \
  memw_update_kernel<C><<<grid, 256, sh, st>>>(nodes, dm.M, dm.dk, dm.d, dm.P, kv, phik, coef, \
                                               A_state, (bf16*)a_act);
  if (chunks <= 4) ARMT_MEMW_CASE(4)
  else if (chunks <= 12) ARMT_MEMW_CASE(12)
  else if (chunks <= 24) ARMT_MEMW_CASE(24)
  else if (chunks <= 32) ARMT_MEMW_CASE(32)
  else return cudaErrorInvalidValue;
#undef ARMT_MEMW_CASE
  return cudaGetLastError();
}

cudaError_t setup_memory_kernels(const Dims& dm) {
  const int sh = (int)(((size_t)dm.M * dm.P + 9 * dm.M) * sizeof(float));
  cudaError_t e = cudaSuccess;
  if (sh > 48 * 1024) {
    e = cudaFuncSetAttribute(memw_update_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, sh);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(memw_update_kernel<12>, cudaFuncAttributeMaxDynamicSharedMemorySize, sh);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(memw_update_kernel<24>, cudaFuncAttributeMaxDynamicSharedMemorySize, sh);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(memw_update_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, sh);
  }
  return e;
}

}  // namespace armt
