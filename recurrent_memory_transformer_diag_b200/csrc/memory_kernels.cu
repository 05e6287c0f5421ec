// ARMT associative-memory write (delta rule) for every node of a wave.
//
// The pages name ARMT as the layer-recurrent model Diagonal Batching targets
// (Pith review of arXiv 2506.05229, "The reading"; each layer updates its
// memory once per segment, "Core claim") and cite the DPFP feature map and
// the delta rule (reference list, refs. 28, 29, 38) without printing them.
// The reading implemented here, for node (s, l): the M memory rows of the
// layer output, RMS-normalised (m_j), give k_j = Wk_mem m_j, v_j = Wv_mem m_j,
// phi_j = DPFP(k_j); the rows are written one after another, j = 0..M-1,
// each seeing the state (A, z) left by the previous rows:
//   vbar_j  = A phi_j / (z . phi_j + eps)
//   gamma_j = clamp(1 - (z . phi_j) / (|phi_j|^2 + eps), 0, 1)
//   A      += (v_j - vbar_j) phi_j^T
//   z      += gamma_j phi_j
//
// Work split.  With z_j the normaliser before row j and G the Gram matrix
// G[j'][j] = phi_j' . phi_j:  z_j . phi_j = z_0 . phi_j + sum_{j'<j} gamma_j' G[j'][j]
// (memw_phi: one block per node, a scalar recurrence after the M dot
// products).  Row i of A: with a the row before the write,
//   (A_j phi_j)[i] = a . phi_j + sum_{j'<j} delta_j' G[j'][j],
//   delta_j = v_j[i] - (A_j phi_j)[i] / (z_j . phi_j + eps),
//   new row = a + sum_j delta_j phi_j
// so memw_update streams A once, row by row (one read, one write per node).
#include "armt_internal.cuh"

namespace armt {

__device__ __forceinline__ float warp_sum_m(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// kv: [slot][M][dk + d] (k first), phik: [slot][M][P], gram: [slot][M][M],
// coef/gamma: [slot][M].  One block per node (one warp per memory row for the
// features, warps over row pairs for the Gram matrix, one thread for the
// M-step recurrence, all threads for the z update).
__global__ void memw_phi_kernel(const NodeEntry* nodes, int M, int dk, int d, int P,
                                const float* kv, float* z_state, float* phik, float* gram, float* coef,
                                float* gamma, float eps) {
  extern __shared__ float sh[];
  const int nw = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* r = sh + warp * 2 * dk;   // [nw][2 dk]
  float* gam = sh + nw * 2 * dk;   // [M]
  float* zp0 = gam + M;            // [M]   z_0 . phi_j
  float* G = zp0 + M;              // [M][M]
  const NodeEntry nd = nodes[blockIdx.x];
  const int slot = nd.z, layer = nd.y;
  float* z = z_state + (long long)layer * P;
  const float* ph_all = phik + (long long)slot * M * P;
  const int n2 = 2 * dk;
  for (int j = warp; j < M; j += nw) {
    const float* k = kv + ((long long)slot * M + j) * (dk + d);
    for (int c = lane; c < dk; c += 32) {
      r[c] = fmaxf(k[c], 0.f);
      r[c + dk] = fmaxf(-k[c], 0.f);
    }
    __syncwarp();
    float* ph = phik + ((long long)slot * M + j) * P;
    float zp = 0.f;
    for (int p = lane; p < P; p += 32) {
      const int n = p / n2 + 1, jj0 = p - (n - 1) * n2;
      int jj = (jj0 - n) % n2;
      if (jj < 0) jj += n2;
      const float f = r[jj0] * r[jj];
      ph[p] = f;
      zp = fmaf(z[p], f, zp);
    }
    zp = warp_sum_m(zp);
    if (lane == 0) zp0[j] = zp;
    __syncwarp();
  }
  __syncthreads();   // phi rows visible block-wide
  for (int pair = warp; pair < M * M; pair += nw) {
    const int a = pair / M, b = pair - a * M;
    if (b < a) continue;
    const float* pa = ph_all + (long long)a * P;
    const float* pb = ph_all + (long long)b * P;
    float g = 0.f;
    for (int p = lane; p < P; p += 32) g = fmaf(pa[p], pb[p], g);
    g = warp_sum_m(g);
    if (lane == 0) {
      G[a * M + b] = g;
      G[b * M + a] = g;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int j = 0; j < M; ++j) {
      float zp = zp0[j];
      for (int jp = 0; jp < j; ++jp) zp = fmaf(gam[jp], G[jp * M + j], zp);
      const float gm = fminf(fmaxf(1.f - zp / (G[j * M + j] + eps), 0.f), 1.f);
      gam[j] = gm;
      coef[(long long)slot * M + j] = 1.f / (zp + eps);
      gamma[(long long)slot * M + j] = gm;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < M * M; e += blockDim.x) gram[(long long)slot * M * M + e] = G[e];
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    float acc = z[p];
    for (int j = 0; j < M; ++j) acc = fmaf(gam[j], ph_all[(long long)j * P + p], acc);
    z[p] = acc;
  }
}

cudaError_t launch_memw_phi(const Dims& dm, const NodeEntry* nodes, int n, const float* kv,
                            float* z_state, float* phik, float* gram, float* coef, float* gamma,
                            cudaStream_t st) {
  const int nw = dm.M < 32 ? dm.M : 32;
  const size_t sh = ((size_t)nw * 2 * dm.dk + 2 * dm.M + (size_t)dm.M * dm.M) * sizeof(float);
  memw_phi_kernel<<<n, nw * 32, sh, st>>>(nodes, dm.M, dm.dk, dm.d, dm.P, kv, z_state, phik, gram, coef,
                                          gamma, dm.mem_eps);
  return cudaGetLastError();
}

constexpr int MEMW_ROWS_PER_BLOCK = 64;

// A_state: [L][d][P] fp32 in place; a_act: optional fp16 copy [L][d][P] (a
// value past the fp16 range sets the error word).
// grid (ceil(d / MEMW_ROWS_PER_BLOCK), nodes), 8 warps, one A row per warp per
// iteration; phi, G and coef are staged once per block.
// Transposed warp reduction of MT per-lane partial sums: afterwards lane l
// holds the warp-wide total of index j = l >> (5 - log2 MT).  Each stage
// halves the values a lane keeps and exchanges the other half with its
// partner (MT - 1 shuffles in the halving stages instead of 5 per index).
template <int K, int O, int MT>
__device__ __forceinline__ void transpose_stage(float (&v)[MT], int lane) {
  if constexpr (O >= 1) {
    if constexpr (K > 1) {
      const bool upper = (lane & O) != 0;
#pragma unroll
      for (int i = 0; i < K / 2; ++i) {
        const float send = upper ? v[i] : v[i + K / 2];
        const float keep = upper ? v[i + K / 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
      }
      transpose_stage<K / 2, O / 2, MT>(v, lane);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
      transpose_stage<1, O / 2, MT>(v, lane);
    }
  }
}

template <int MT>
__device__ __forceinline__ float transpose_reduce(float (&v)[MT], int lane) {
  transpose_stage<MT, 16, MT>(v, lane);
  return v[0];
}

template <int MT>
constexpr int log2_const() { return MT <= 1 ? 0 : 1 + log2_const<MT / 2>(); }

// M <= MT <= 32: lane j carries memory row j through the recurrence.  A warp
// updates R = 2 rows of A per pass (rows i and i + 8 of its block's range), so
// every phi element read from shared memory serves both rows (R = 4 measured
// slower: 212 registers leave one block per SM).
constexpr int MEMW_R = 2;

template <int MAXC, int MT>
__global__ void __launch_bounds__(256) memw_update_kernel(const NodeEntry* nodes, int M, int dk, int d, int P,
                                                          const float* kv, const float* phik,
                                                          const float* gram, const float* coef, float* A_state,
                                                          f16* a_act, unsigned* err) {
  constexpr int R = MEMW_R;
  extern __shared__ float sh[];
  float* ph = sh;                    // [M][P]
  float* G = ph + M * P;             // [M][M]
  float* cf = G + M * M;             // [M]
  float* dots = cf + M;              // [8][R][M]  delta_j per warp and row
  const NodeEntry nd = nodes[blockIdx.y];
  const int slot = nd.z, layer = nd.y;
  for (int e = threadIdx.x; e < M * P; e += blockDim.x) ph[e] = phik[(long long)slot * M * P + e];
  for (int e = threadIdx.x; e < M * M; e += blockDim.x) G[e] = gram[(long long)slot * M * M + e];
  for (int e = threadIdx.x; e < M; e += blockDim.x) cf[e] = coef[(long long)slot * M + e];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* dl = dots + warp * R * M;
  bool over = false;
  constexpr int SHIFT = 5 - log2_const<MT>();
  const float cj = lane < M ? cf[lane] : 0.f;
  const int i_begin = blockIdx.x * MEMW_ROWS_PER_BLOCK;
  const int i_end = min(d, i_begin + MEMW_ROWS_PER_BLOCK);
  const float* kvj = kv + ((long long)slot * M + (lane < M ? lane : 0)) * (dk + d) + dk;
  for (int i0 = i_begin + warp; i0 < i_end; i0 += 8 * R) {
    float a[R][MAXC];
    float v[R];
    bool has[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = i0 + 8 * r;
      has[r] = i < i_end;
      const float* Arow = A_state + ((long long)layer * d + (has[r] ? i : i0)) * P;
      v[r] = (lane < M && has[r]) ? kvj[i] : 0.f;
#pragma unroll
      for (int c = 0; c < MAXC; ++c) {
        const int p = lane + 32 * c;
        a[r][c] = (p < P && has[r]) ? Arow[p] : 0.f;
      }
    }
    // a_r . phi_j for all rows and j at once (independent accumulators)
    float part[R][MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int j = 0; j < MT; ++j) part[r][j] = 0.f;
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int p = lane + 32 * c;
      if (p < P) {
#pragma unroll
        for (int j = 0; j < MT; ++j) {
          if (j < M) {
            const float f = ph[j * P + p];
#pragma unroll
            for (int r = 0; r < R; ++r) part[r][j] = fmaf(a[r][c], f, part[r][j]);
          }
        }
      }
    }
    // lane j (< M) keeps s_j = a . phi_j + sum_{j'<j} delta_j' G[j'][j]
    float sv[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float tot = transpose_reduce<MT>(part[r], lane);
      sv[r] = __shfl_sync(0xffffffffu, tot, (lane << SHIFT) & 31);
    }
    for (int j = 0; j < M; ++j) {
      // delta_j = v_j[i] - s_j coef_j; s_j is final once rows 0..j-1 are applied
      const float gj = (lane > j && lane < M) ? G[j * M + lane] : 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float dj = __shfl_sync(0xffffffffu, v[r] - sv[r] * cj, j);
        if (lane == j) dl[r * M + j] = dj;
        sv[r] = fmaf(dj, gj, sv[r]);
      }
    }
    __syncwarp();
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int p = lane + 32 * c;
      if (p < P) {
        float acc[R];
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r] = a[r][c];
        for (int j = 0; j < M; ++j) {
          const float f = ph[j * P + p];
#pragma unroll
          for (int r = 0; r < R; ++r) acc[r] = fmaf(dl[r * M + j], f, acc[r]);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          if (!has[r]) continue;
          const long long off = ((long long)layer * d + i0 + 8 * r) * P + p;
          A_state[off] = acc[r];
          if (a_act) {
            a_act[off] = __float2half_rn(acc[r]);
            over |= fabsf(acc[r]) > 65504.f;
          }
        }
      }
    }
    __syncwarp();
  }
  if (err && __any_sync(0xffffffffu, over) && lane == 0) atomicOr(err, ERR_FP16_RANGE);
}

// Same computation with 16-byte accesses (P % 4 == 0): lane l owns the
// column groups 4 (l + 32 c) .. +3, c < C4, so A rows are read and written as
// float4 and every phi read from shared memory is one 16-byte load serving
// 4 columns of both rows.  At most 128 registers: two blocks per SM.
template <int C4, int MT>
__global__ void __launch_bounds__(256, 2) memw_update_vec_kernel(const NodeEntry* nodes, int M, int dk, int d, int P,
                                                                 const float* kv, const float* phik,
                                                                 const float* gram, const float* coef,
                                                                 float* A_state, f16* a_act, unsigned* err) {
  constexpr int R = MEMW_R;
  extern __shared__ float sh[];
  float* ph = sh;                    // [M][P]
  float* G = ph + M * P;             // [M][M]
  float* cf = G + M * M;             // [M]
  float* dots = cf + M;              // [8][R][M]  delta_j per warp and row
  const NodeEntry nd = nodes[blockIdx.y];
  const int slot = nd.z, layer = nd.y;
  const int P4 = P >> 2;
  {
    const float4* src = reinterpret_cast<const float4*>(phik + (long long)slot * M * P);
    float4* dst = reinterpret_cast<float4*>(ph);
    for (int e = threadIdx.x; e < M * P4; e += blockDim.x) dst[e] = src[e];
  }
  for (int e = threadIdx.x; e < M * M; e += blockDim.x) G[e] = gram[(long long)slot * M * M + e];
  for (int e = threadIdx.x; e < M; e += blockDim.x) cf[e] = coef[(long long)slot * M + e];
  __syncthreads();
  const float4* ph4 = reinterpret_cast<const float4*>(ph);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* dl = dots + warp * R * M;
  bool over = false;
  constexpr int SHIFT = 5 - log2_const<MT>();
  const float cj = lane < M ? cf[lane] : 0.f;
  const int i_begin = blockIdx.x * MEMW_ROWS_PER_BLOCK;
  const int i_end = min(d, i_begin + MEMW_ROWS_PER_BLOCK);
  const float* kvj = kv + ((long long)slot * M + (lane < M ? lane : 0)) * (dk + d) + dk;
  for (int i0 = i_begin + warp; i0 < i_end; i0 += 8 * R) {
    float4 a[R][C4];
    float v[R];
    bool has[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = i0 + 8 * r;
      has[r] = i < i_end;
      const float4* Arow = reinterpret_cast<const float4*>(A_state + ((long long)layer * d + (has[r] ? i : i0)) * P);
      v[r] = (lane < M && has[r]) ? kvj[i] : 0.f;
#pragma unroll
      for (int c = 0; c < C4; ++c) {
        const int q = lane + 32 * c;
        a[r][c] = (q < P4 && has[r]) ? Arow[q] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    // a_r . phi_j for all rows and j at once (independent accumulators)
    float part[R][MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int j = 0; j < MT; ++j) part[r][j] = 0.f;
#pragma unroll
    for (int c = 0; c < C4; ++c) {
      const int q = lane + 32 * c;
      if (q < P4) {
#pragma unroll
        for (int j = 0; j < MT; ++j) {
          if (j < M) {
            const float4 f = ph4[j * P4 + q];
#pragma unroll
            for (int r = 0; r < R; ++r) {
              float t = fmaf(a[r][c].x, f.x, part[r][j]);
              t = fmaf(a[r][c].y, f.y, t);
              t = fmaf(a[r][c].z, f.z, t);
              part[r][j] = fmaf(a[r][c].w, f.w, t);
            }
          }
        }
      }
    }
    // lane j (< M) keeps s_j = a . phi_j + sum_{j'<j} delta_j' G[j'][j]
    float sv[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float tot = transpose_reduce<MT>(part[r], lane);
      sv[r] = __shfl_sync(0xffffffffu, tot, (lane << SHIFT) & 31);
    }
    for (int j = 0; j < M; ++j) {
      // delta_j = v_j[i] - s_j coef_j; s_j is final once rows 0..j-1 are applied
      const float gj = (lane > j && lane < M) ? G[j * M + lane] : 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float dj = __shfl_sync(0xffffffffu, v[r] - sv[r] * cj, j);
        if (lane == j) dl[r * M + j] = dj;
        sv[r] = fmaf(dj, gj, sv[r]);
      }
    }
    __syncwarp();
#pragma unroll
    for (int c = 0; c < C4; ++c) {
      const int q = lane + 32 * c;
      if (q < P4) {
        float4 acc[R];
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r] = a[r][c];
        for (int j = 0; j < M; ++j) {
          const float4 f = ph4[j * P4 + q];
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const float dj = dl[r * M + j];
            acc[r].x = fmaf(dj, f.x, acc[r].x);
            acc[r].y = fmaf(dj, f.y, acc[r].y);
            acc[r].z = fmaf(dj, f.z, acc[r].z);
            acc[r].w = fmaf(dj, f.w, acc[r].w);
          }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          if (!has[r]) continue;
          const long long off = ((long long)layer * d + i0 + 8 * r) * P + 4 * q;
          *reinterpret_cast<float4*>(A_state + off) = acc[r];
          if (a_act) {
            const __half2 lo = __floats2half2_rn(acc[r].x, acc[r].y), hi = __floats2half2_rn(acc[r].z, acc[r].w);
            uint2 pk;
            pk.x = *reinterpret_cast<const uint32_t*>(&lo);
            pk.y = *reinterpret_cast<const uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(a_act + off) = pk;
            over |= fmaxf(fmaxf(fabsf(acc[r].x), fabsf(acc[r].y)), fmaxf(fabsf(acc[r].z), fabsf(acc[r].w))) > 65504.f;
          }
        }
      }
    }
    __syncwarp();
  }
  if (err && __any_sync(0xffffffffu, over) && lane == 0) atomicOr(err, ERR_FP16_RANGE);
}

static size_t memw_update_smem(const Dims& dm) {
  return ((size_t)dm.M * dm.P + (size_t)dm.M * dm.M + dm.M + 8 * MEMW_R * dm.M) * sizeof(float);
}

cudaError_t launch_memw_update(const Dims& dm, const NodeEntry* nodes, int n, const float* kv,
                               const float* phik, const float* gram, const float* coef, float* A_state,
                               void* a_act, unsigned* err, cudaStream_t st) {
  dim3 grid((dm.d + MEMW_ROWS_PER_BLOCK - 1) / MEMW_ROWS_PER_BLOCK, n);
  const size_t sh = memw_update_smem(dm);
  const int chunks = (dm.P + 31) / 32;
#define ARMT_MEMW_CASE(C, MT)                                                                             \
  memw_update_kernel<C, MT><<<grid, 256, sh, st>>>(nodes, dm.M, dm.dk, dm.d, dm.P, kv, phik, gram, coef, \
                                                   A_state, (f16*)a_act, err);
#define ARMT_MEMW_M(C)                  \
  {                                     \
    if (dm.M <= 4) ARMT_MEMW_CASE(C, 4) \
    else if (dm.M <= 16) ARMT_MEMW_CASE(C, 16) \
    else ARMT_MEMW_CASE(C, 32)          \
  }
  if (dm.M > 32) return cudaErrorInvalidValue;
  if (dm.P % 4 == 0 && dm.P <= 1024) {   // 16-byte path
    const int c4 = (dm.P / 4 + 31) / 32;
#define ARMT_MEMWV_CASE(C, MT)                                                                                \
  memw_update_vec_kernel<C, MT><<<grid, 256, sh, st>>>(nodes, dm.M, dm.dk, dm.d, dm.P, kv, phik, gram, coef, \
                                                       A_state, (f16*)a_act, err);
#define ARMT_MEMWV_M(C)                  \
  {                                      \
    if (dm.M <= 4) ARMT_MEMWV_CASE(C, 4) \
    else if (dm.M <= 16) ARMT_MEMWV_CASE(C, 16) \
    else ARMT_MEMWV_CASE(C, 32)          \
  }
    if (c4 <= 2) ARMT_MEMWV_M(2)
    else if (c4 <= 3) ARMT_MEMWV_M(3)
    else if (c4 <= 4) ARMT_MEMWV_M(4)
    else if (c4 <= 6) ARMT_MEMWV_M(6)
    else ARMT_MEMWV_M(8)
#undef ARMT_MEMWV_M
#undef ARMT_MEMWV_CASE
    return cudaGetLastError();
  }
  if (chunks <= 4) ARMT_MEMW_M(4)
  else if (chunks <= 12) ARMT_MEMW_M(12)
  else if (chunks <= 24) ARMT_MEMW_M(24)
  else if (chunks <= 32) ARMT_MEMW_M(32)
  else return cudaErrorInvalidValue;
#undef ARMT_MEMW_M
#undef ARMT_MEMW_CASE
  return cudaGetLastError();
}

cudaError_t setup_memory_kernels(const Dims& dm) {
  const int sh = (int)memw_update_smem(dm);
  cudaError_t e = cudaSuccess;
  if (sh > 48 * 1024) {
    auto set = [&](auto fn) {
      if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, sh);
    };
    set(memw_update_kernel<4, 4>); set(memw_update_kernel<4, 16>); set(memw_update_kernel<4, 32>);
    set(memw_update_kernel<12, 4>); set(memw_update_kernel<12, 16>); set(memw_update_kernel<12, 32>);
    set(memw_update_kernel<24, 4>); set(memw_update_kernel<24, 16>); set(memw_update_kernel<24, 32>);
    set(memw_update_kernel<32, 4>); set(memw_update_kernel<32, 16>); set(memw_update_kernel<32, 32>);
    set(memw_update_vec_kernel<2, 4>); set(memw_update_vec_kernel<2, 16>); set(memw_update_vec_kernel<2, 32>);
    set(memw_update_vec_kernel<3, 4>); set(memw_update_vec_kernel<3, 16>); set(memw_update_vec_kernel<3, 32>);
    set(memw_update_vec_kernel<4, 4>); set(memw_update_vec_kernel<4, 16>); set(memw_update_vec_kernel<4, 32>);
    set(memw_update_vec_kernel<6, 4>); set(memw_update_vec_kernel<6, 16>); set(memw_update_vec_kernel<6, 32>);
    set(memw_update_vec_kernel<8, 4>); set(memw_update_vec_kernel<8, 16>); set(memw_update_vec_kernel<8, 32>);
  }
  return e;
}

}  // namespace armt
