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
//   A      += beta_j (v_j - vbar_j) phi_j^T
//   z      += gamma_j phi_j
// with beta_j = 1, or, for the gated write, beta_j = sigmoid(w_beta . m_j)
// (the projection's extra output column); gamma_j may also be left unclamped.
//
// Work split.  With z_j the normaliser before row j and G the Gram matrix
// G[j'][j] = phi_j' . phi_j:  z_j . phi_j = z_0 . phi_j + sum_{j'<j} gamma_j' G[j'][j]
// (memw_phi: one block per node, a scalar recurrence after the M dot
// products).  Row i of A: with a the row before the write,
//   (A_j phi_j)[i] = a . phi_j + sum_{j'<j} delta_j' G[j'][j],
//   delta_j = beta_j (v_j[i] - (A_j phi_j)[i] / (z_j . phi_j + eps)),
//   new row = a + sum_j delta_j phi_j
// so memw_update streams A once, row by row (one read, one write per node).
#include "armt_internal.cuh"

namespace armt {

__device__ __forceinline__ float warp_sum_m(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// kv: [slot][M][ldkv] rows [k (dk) | v (d) | gate logit (gated write)],
// phik: [slot][M][P], gram: [slot][M][M], coef/gamma/beta: [slot][M].  One
// block per node: one warp per memory row for the features (phi kept in
// shared memory for the Gram matrix), warps over row pairs for the Gram
// matrix, one warp for the M-step recurrence, all threads for the z update.
__global__ void memw_phi_kernel(const NodeEntry* nodes, int M, int dk, int d, int P, int nu, int ldkv,
                                const float* kv, float* z_state, float* phik, float* gram, float* coef,
                                float* gamma, float* beta, int clamp_gamma, float eps) {
  grid_dependency_sync();
  extern __shared__ float sh[];
  const int nw = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n2 = 2 * dk;
  float* zs = sh;                  // [P]     z before the write
  float* phs = zs + P;             // [M][P]  phi_j
  float* r = phs + M * P;          // [nw][2 dk]
  float* gam = r + nw * n2;        // [M]
  float* zp0 = gam + M;            // [M]     z_0 . phi_j
  float* G = zp0 + M;              // [M][M]
  const NodeEntry nd = nodes[blockIdx.x];
  const int slot = nd.z, layer = nd.y;
  float* z = z_state + (long long)layer * P;
  for (int p = threadIdx.x; p < P; p += blockDim.x) zs[p] = z[p];
  __syncthreads();
  for (int j = warp; j < M; j += nw) {
    const float* k = kv + ((long long)slot * M + j) * ldkv;
    if (beta && lane == 0) beta[(long long)slot * M + j] = 1.f / (1.f + __expf(-k[dk + d]));
    float* rw = r + warp * n2;
    for (int c = lane; c < dk; c += 32) {
      const float kc = k[c];
      rw[c] = fmaxf(kc, 0.f);
      rw[c + dk] = fmaxf(-kc, 0.f);
    }
    __syncwarp();
    float* phj = phs + j * P;
    float* phg = phik + ((long long)slot * M + j) * P;
    float zp = 0.f;
    for (int n = 1; n <= nu; ++n) {      // block n: r_i * r_{(i - n) mod 2dk} (nu <= 2 dk)
      for (int i = lane; i < n2; i += 32) {
        const int i2 = i - n < 0 ? i - n + n2 : i - n;
        const float f = rw[i] * rw[i2];
        const int p = (n - 1) * n2 + i;
        phj[p] = f;
        phg[p] = f;
        zp = fmaf(zs[p], f, zp);
      }
    }
    zp = warp_sum_m(zp);
    if (lane == 0) zp0[j] = zp;
    __syncwarp();
  }
  __syncthreads();   // phi rows visible block-wide
  // Gram matrix: the M (M + 1) / 2 pairs a <= b, dealt to the warps; each dot
  // product keeps four partial sums (a short dependency chain)
  for (int q = warp; q < M * (M + 1) / 2; q += nw) {
    int a = 0, rest = q;
    while (rest >= M - a) { rest -= M - a; ++a; }
    const int b = a + rest;
    const float* pa = phs + a * P;
    const float* pb = phs + b * P;
    float g0 = 0.f, g1 = 0.f, g2 = 0.f, g3 = 0.f;
    int p = lane;
    for (; p + 96 < P; p += 128) {
      g0 = fmaf(pa[p], pb[p], g0);
      g1 = fmaf(pa[p + 32], pb[p + 32], g1);
      g2 = fmaf(pa[p + 64], pb[p + 64], g2);
      g3 = fmaf(pa[p + 96], pb[p + 96], g3);
    }
    for (; p < P; p += 32) g0 = fmaf(pa[p], pb[p], g0);
    const float g = warp_sum_m((g0 + g1) + (g2 + g3));
    if (lane == 0) {
      G[a * M + b] = g;
      G[b * M + a] = g;
    }
  }
  __syncthreads();
  if (warp == 0) {
    // z_j . phi_j = z_0 . phi_j + sum_{j'<j} gamma_j' G[j'][j]: lane j (< M <= 32)
    // carries row j; at step j lane j's value is final, gamma_j is broadcast
    // and the later lanes add its term.  Lane j's denominator |phi_j|^2 + eps
    // and its column of G are read once, before the steps.
    const int jl = lane < M ? lane : 0;
    const float den = G[jl * (M + 1)] + eps;
    float gcol[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) gcol[j] = (j < M) ? G[j * M + jl] : 0.f;
    float zp = lane < M ? zp0[lane] : 0.f;
    float gm_own = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j < M) {
        const float g_raw = 1.f - zp / den;
        const float gm_l = clamp_gamma ? fminf(fmaxf(g_raw, 0.f), 1.f) : g_raw;
        const float gm = __shfl_sync(0xffffffffu, gm_l, j);
        if (lane == j) gm_own = gm;
        if (lane > j) zp = fmaf(gm, gcol[j], zp);
      }
    }
    // zp is lane j's final z_j . phi_j (no step after j changes it)
    if (lane < M) {
      gam[lane] = gm_own;
      coef[(long long)slot * M + lane] = 1.f / (zp + eps);
      gamma[(long long)slot * M + lane] = gm_own;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < M * M; e += blockDim.x) gram[(long long)slot * M * M + e] = G[e];
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    float a0 = zs[p], a1 = 0.f;
    int j = 0;
    for (; j + 1 < M; j += 2) {
      a0 = fmaf(gam[j], phs[j * P + p], a0);
      a1 = fmaf(gam[j + 1], phs[(j + 1) * P + p], a1);
    }
    if (j < M) a0 = fmaf(gam[j], phs[j * P + p], a0);
    z[p] = a0 + a1;
  }
}

size_t memw_phi_smem(const Dims& dm) {
  const int nw = dm.M < 32 ? dm.M : 32;
  return ((size_t)dm.P + (size_t)dm.M * dm.P + (size_t)nw * 2 * dm.dk + 2 * dm.M + (size_t)dm.M * dm.M) *
         sizeof(float);
}

cudaError_t launch_memw_phi(const Dims& dm, const NodeEntry* nodes, int n, const float* kv,
                            float* z_state, float* phik, float* gram, float* coef, float* gamma, float* beta,
                            cudaStream_t st) {
  const int nw = dm.M < 32 ? dm.M : 32;
  return launch_pdl(memw_phi_kernel, dim3(n), dim3(nw * 32), memw_phi_smem(dm), st, nodes, dm.M, dm.dk, dm.d, dm.P,
                    dm.nu, kv_ld(dm), kv, z_state, phik, gram, coef, gamma, dm.write_gate ? beta : nullptr,
                    dm.clamp_gamma ? 1 : 0, dm.mem_eps);
}

constexpr int MEMW_ROWS_PER_BLOCK = 64;

// A_state: [L][d][P] fp32 in place.
// grid (ceil(d / MEMW_ROWS_PER_BLOCK), nodes), 8 warps, one A row per warp per
// iteration; phi, G, coef and beta are staged once per block.
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
                                                          int ldkv, const float* kv, const float* phik,
                                                          const float* gram, const float* coef, const float* beta,
                                                          float* A_state) {
  grid_dependency_sync();
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
  constexpr int SHIFT = 5 - log2_const<MT>();
  const float cj = lane < M ? cf[lane] : 0.f;
  const float bj = (beta && lane < M) ? beta[(long long)slot * M + lane] : 1.f;
  const int i_begin = blockIdx.x * MEMW_ROWS_PER_BLOCK;
  const int i_end = min(d, i_begin + MEMW_ROWS_PER_BLOCK);
  const float* kvj = kv + ((long long)slot * M + (lane < M ? lane : 0)) * ldkv + dk;
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
        const float dj = __shfl_sync(0xffffffffu, bj * (v[r] - sv[r] * cj), j);
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
          A_state[((long long)layer * d + i0 + 8 * r) * P + p] = acc[r];
        }
      }
    }
    __syncwarp();
  }
}

// Same computation with 16-byte accesses (P % 4 == 0): lane l owns the
// column groups 4 (l + 32 c) .. +3, c < C4, so A rows are read and written as
// float4 and every phi read from shared memory is one 16-byte load serving
// 4 columns of both rows.  At most 128 registers: two blocks per SM.  With
// PF, each warp's next two rows are copied into shared memory (cp.async, a
// two-buffer ring per warp) while it works on the current two, so the A
// stream's latency overlaps the arithmetic.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int C4, int MT, bool PF>
__global__ void __launch_bounds__(256, 2) memw_update_vec_kernel(const NodeEntry* nodes, int M, int dk, int d, int P,
                                                                 int ldkv, const float* kv, const float* phik,
                                                                 const float* gram, const float* coef,
                                                                 const float* beta, float* A_state) {
  grid_dependency_sync();
  constexpr int R = MEMW_R;
  extern __shared__ float sh[];
  float* ph = sh;                    // [M][P]
  float* G = ph + M * P;             // [M][M]
  float* cf = G + M * M;             // [M]
  // (the next 8 R M floats are unused here: the layout matches the scalar kernel's)
  float* pf = sh + ((M * P + M * M + M + 8 * R * M + 3) & ~3);   // PF: [8 warps][2][R][P] rows of A in flight (16-byte aligned)
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
  constexpr int SHIFT = 5 - log2_const<MT>();
  const float cj = lane < M ? cf[lane] : 0.f;
  const float bj = (beta && lane < M) ? beta[(long long)slot * M + lane] : 1.f;
  const int i_begin = blockIdx.x * MEMW_ROWS_PER_BLOCK;
  const int i_end = min(d, i_begin + MEMW_ROWS_PER_BLOCK);
  const float* kvj = kv + ((long long)slot * M + (lane < M ? lane : 0)) * ldkv + dk;
  // rows i0n + 8 r of this warp -> buffer b (each lane copies the 16-byte
  // groups it later reads itself)
  auto issue_rows = [&](int i0n, int b) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = i0n + 8 * r;
      if (i < i_end) {
        const float* src = A_state + ((long long)layer * d + i) * P;
        float* dst = pf + ((warp * 2 + b) * R + r) * P;
#pragma unroll
        for (int c = 0; c < C4; ++c) {
          const int q = lane + 32 * c;
          if (q < P4) cp_async16(dst + 4 * q, src + 4 * q);
        }
      }
    }
    cp_async_commit();
  };
  int buf = 0;
  if (PF) issue_rows(i_begin + warp, 0);
  for (int i0 = i_begin + warp; i0 < i_end; i0 += 8 * R) {
    float4 a[R][C4];
    float v[R];
    bool has[R];
    if (PF) {
      issue_rows(i0 + 8 * R, buf ^ 1);   // the next pass (an empty group past the end)
      cp_async_wait<1>();                // this pass's rows have landed
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = i0 + 8 * r;
      has[r] = i < i_end;
      const float4* Arow = PF ? reinterpret_cast<const float4*>(pf + ((warp * 2 + buf) * R + r) * P)
                              : reinterpret_cast<const float4*>(A_state + ((long long)layer * d + (has[r] ? i : i0)) * P);
      v[r] = (lane < M && has[r]) ? kvj[i] : 0.f;
#pragma unroll
      for (int c = 0; c < C4; ++c) {
        const int q = lane + 32 * c;
        a[r][c] = (q < P4 && has[r]) ? Arow[q] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    buf ^= 1;
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
    // every lane receives each delta_j as it is broadcast, so the deltas stay
    // in registers for the update (no shared-memory round trip)
    float dreg[R][MT];
#pragma unroll
    for (int j = 0; j < MT; ++j) {
      if (j < M) {
        // delta_j = v_j[i] - s_j coef_j; s_j is final once rows 0..j-1 are applied
        const float gj = (lane > j && lane < M) ? G[j * M + lane] : 0.f;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float dj = __shfl_sync(0xffffffffu, bj * (v[r] - sv[r] * cj), j);
          dreg[r][j] = dj;
          sv[r] = fmaf(dj, gj, sv[r]);
        }
      } else {
#pragma unroll
        for (int r = 0; r < R; ++r) dreg[r][j] = 0.f;
      }
    }
#pragma unroll
    for (int c = 0; c < C4; ++c) {
      const int q = lane + 32 * c;
      if (q < P4) {
        float4 acc[R];
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r] = a[r][c];
#pragma unroll
        for (int j = 0; j < MT; ++j) {
          if (j < M) {
            const float4 f = ph4[j * P4 + q];
#pragma unroll
            for (int r = 0; r < R; ++r) {
              const float dj = dreg[r][j];
              acc[r].x = fmaf(dj, f.x, acc[r].x);
              acc[r].y = fmaf(dj, f.y, acc[r].y);
              acc[r].z = fmaf(dj, f.z, acc[r].z);
              acc[r].w = fmaf(dj, f.w, acc[r].w);
            }
          }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          if (!has[r]) continue;
          *reinterpret_cast<float4*>(A_state + ((long long)layer * d + i0 + 8 * r) * P + 4 * q) = acc[r];
        }
      }
    }
    __syncwarp();
  }
  if (PF) cp_async_wait<0>();
}

static size_t memw_update_smem(const Dims& dm) {
  return ((size_t)dm.M * dm.P + (size_t)dm.M * dm.M + dm.M + 8 * MEMW_R * dm.M) * sizeof(float);
}

// with the per-warp two-buffer ring of A rows; used when two blocks still fit on an SM
static size_t memw_update_pf_smem(const Dims& dm) {
  const size_t base = ((size_t)dm.M * dm.P + (size_t)dm.M * dm.M + dm.M + 8 * MEMW_R * dm.M + 3) & ~(size_t)3;
  return (base + (size_t)8 * 2 * MEMW_R * dm.P) * sizeof(float);
}
constexpr size_t MEMW_PF_SMEM_MAX = 110 * 1024;

cudaError_t launch_memw_update(const Dims& dm, const NodeEntry* nodes, int n, const float* kv,
                               const float* phik, const float* gram, const float* coef, const float* beta,
                               float* A_state, cudaStream_t st) {
  const int ldkv = kv_ld(dm);
  if (!dm.write_gate) beta = nullptr;
  dim3 grid((dm.d + MEMW_ROWS_PER_BLOCK - 1) / MEMW_ROWS_PER_BLOCK, n);
  const size_t sh = memw_update_smem(dm);
  const int chunks = (dm.P + 31) / 32;
#define ARMT_MEMW_CASE(C, MT)                                                                             \
  memw_update_kernel<C, MT><<<grid, 256, sh, st>>>(nodes, dm.M, dm.dk, dm.d, dm.P, ldkv, kv, phik, gram, coef, \
                                                   beta, A_state);
#define ARMT_MEMW_M(C)                  \
  {                                     \
    if (dm.M <= 4) ARMT_MEMW_CASE(C, 4) \
    else if (dm.M <= 16) ARMT_MEMW_CASE(C, 16) \
    else ARMT_MEMW_CASE(C, 32)          \
  }
  if (dm.M > 32) return cudaErrorInvalidValue;
  // the 16-byte kernel reads and writes A rows and reads the phi rows as
  // float4: both bases must be 16-byte aligned
  const bool aligned = (reinterpret_cast<uintptr_t>(A_state) & 15) == 0 &&
                       (reinterpret_cast<uintptr_t>(phik) & 15) == 0;
  if (dm.P % 4 == 0 && dm.P <= 1024 && aligned) {   // 16-byte path
    const int c4 = (dm.P / 4 + 31) / 32;
    const size_t sh_pf = memw_update_pf_smem(dm);
    const bool pf = sh_pf <= MEMW_PF_SMEM_MAX;
    cudaError_t e = cudaSuccess;
#define ARMT_MEMWV_CASE(C, MT)                                                                                      \
  {                                                                                                                 \
    if (pf)                                                                                                         \
      e = launch_pdl(memw_update_vec_kernel<C, MT, true>, grid, dim3(256), sh_pf, st, nodes, dm.M, dm.dk,     \
                     dm.d, dm.P, ldkv, kv, phik, gram, coef, beta, A_state);                                        \
    else                                                                                                            \
      e = launch_pdl(memw_update_vec_kernel<C, MT, false>, grid, dim3(256), sh, st, nodes, dm.M, dm.dk, dm.d,   \
                     dm.P, ldkv, kv, phik, gram, coef, beta, A_state);                                              \
  }
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
    return e;
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
  if (memw_phi_smem(dm) > 48 * 1024)
    e = cudaFuncSetAttribute(memw_phi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)memw_phi_smem(dm));
  if (sh > 48 * 1024) {
    auto set = [&](auto fn) {
      if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, sh);
    };
    set(memw_update_kernel<4, 4>); set(memw_update_kernel<4, 16>); set(memw_update_kernel<4, 32>);
    set(memw_update_kernel<12, 4>); set(memw_update_kernel<12, 16>); set(memw_update_kernel<12, 32>);
    set(memw_update_kernel<24, 4>); set(memw_update_kernel<24, 16>); set(memw_update_kernel<24, 32>);
    set(memw_update_kernel<32, 4>); set(memw_update_kernel<32, 16>); set(memw_update_kernel<32, 32>);
    set(memw_update_vec_kernel<2, 4, false>); set(memw_update_vec_kernel<2, 16, false>); set(memw_update_vec_kernel<2, 32, false>);
    set(memw_update_vec_kernel<3, 4, false>); set(memw_update_vec_kernel<3, 16, false>); set(memw_update_vec_kernel<3, 32, false>);
    set(memw_update_vec_kernel<4, 4, false>); set(memw_update_vec_kernel<4, 16, false>); set(memw_update_vec_kernel<4, 32, false>);
    set(memw_update_vec_kernel<6, 4, false>); set(memw_update_vec_kernel<6, 16, false>); set(memw_update_vec_kernel<6, 32, false>);
    set(memw_update_vec_kernel<8, 4, false>); set(memw_update_vec_kernel<8, 16, false>); set(memw_update_vec_kernel<8, 32, false>);
  }
  const size_t sh_pf = memw_update_pf_smem(dm);
  if (sh_pf <= MEMW_PF_SMEM_MAX && sh_pf > 48 * 1024) {
    auto set = [&](auto fn) {
      if (e == cudaSuccess) e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sh_pf);
    };
    set(memw_update_vec_kernel<2, 4, true>); set(memw_update_vec_kernel<2, 16, true>); set(memw_update_vec_kernel<2, 32, true>);
    set(memw_update_vec_kernel<3, 4, true>); set(memw_update_vec_kernel<3, 16, true>); set(memw_update_vec_kernel<3, 32, true>);
    set(memw_update_vec_kernel<4, 4, true>); set(memw_update_vec_kernel<4, 16, true>); set(memw_update_vec_kernel<4, 32, true>);
    set(memw_update_vec_kernel<6, 4, true>); set(memw_update_vec_kernel<6, 16, true>); set(memw_update_vec_kernel<6, 32, true>);
    set(memw_update_vec_kernel<8, 4, true>); set(memw_update_vec_kernel<8, 16, true>); set(memw_update_vec_kernel<8, 32, true>);
  }
  return e;
}

}  // namespace armt
