// SIMT kernels of the forward: the fp32 path end to end, and the row-wise
// steps (layer-0 input, RMSNorm, DPFP features, output) of the tensor-core path.
//
// Every kernel takes the wave's node entries (segment, layer, slot) and
// handles all nodes of the wave in one launch (blockIdx.z or blockIdx.y =
// node), which is what turns S x L node steps into S + L - 1 grouped steps
// ("Diagonal Batching for Recurrent Memory Transformers" skill page,
// "Architecture Overview": one grouped kernel launch per diagonal).
#include "armt_internal.cuh"

namespace armt {

__device__ __forceinline__ float ld(const float* p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld(const bf16* p, size_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void st(float* p, size_t i, float v) { p[i] = v; }
__device__ __forceinline__ void st(bf16* p, size_t i, float v) { p[i] = __float2bfloat16_rn(v); }
__device__ __forceinline__ float ld(const f16* p, size_t i) { return __half2float(p[i]); }
__device__ __forceinline__ void st(f16* p, size_t i, float v) { p[i] = __float2half_rn(v); }
// v as stored in an array of T (rounded to T's precision)
template <typename T> __device__ __forceinline__ float rounded(float v);
template <> __device__ __forceinline__ float rounded<float>(float v) { return v; }
template <> __device__ __forceinline__ float rounded<f16>(float v) { return __half2float(__float2half_rn(v)); }
template <> __device__ __forceinline__ float rounded<bf16>(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// Grouped GEMM, SIMT: C[node] = A[node] (M x K) * B[layer(node)]^T (B is N x K)
// 64x64 tile per block, 256 threads, 4x4 outputs per thread, fp32 accumulate.
// ---------------------------------------------------------------------------
template <typename TA, typename TB, typename TC>
__global__ void __launch_bounds__(256) simt_gemm_kernel(GemmArgs g) {
  const NodeEntry nd = g.nodes[blockIdx.z];
  const int layer = nd.y, slot = nd.z;
  const TA* A = reinterpret_cast<const TA*>(g.A) + (long long)(g.a_by_layer ? layer : slot) * g.a_slot_stride;
  const TB* B = reinterpret_cast<const TB*>(g.B) + (long long)layer * g.b_layer_stride;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  if (m0 >= g.M) return;
  __shared__ float As[16][68];
  __shared__ float Bs[16][68];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < g.K; k0 += 16) {
    for (int e = threadIdx.x; e < 1024; e += 256) {
      const int r = e >> 4, kk = e & 15;
      const int gk = k0 + kk;
      const int ga = m0 + r, gb = n0 + r;
      As[kk][r] = (ga < g.M && gk < g.K) ? ld(A, (size_t)ga * g.lda + gk) : 0.f;
      Bs[kk][r] = (gb < g.N && gk < g.K) ? ld(B, (size_t)gb * g.ldb + gk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  const long long coff = (long long)slot * g.c_slot_stride;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = m0 + ty + 16 * i;
    if (row >= g.M) continue;
    const float rs = g.rowscale ? g.rowscale[(long long)slot * g.rs_slot_stride + row] : 1.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = n0 + tx + 16 * j;
      if (col >= g.N) continue;
      const float v = acc[i][j] * rs;
      const size_t idx = coff + (size_t)row * g.ldc + col;
      if (g.epi == EPI_RESID) {
        float* C = reinterpret_cast<float*>(g.C);
        C[idx] += v;
      } else {
        st(reinterpret_cast<TC*>(g.C), idx, v);
      }
    }
  }
}

cudaError_t launch_simt_gemm(const GemmArgs& a, cudaStream_t st) {
  if (a.n_nodes <= 0) return cudaSuccess;
  dim3 grid((a.N + 63) / 64, (a.M + 63) / 64, a.n_nodes);
  simt_gemm_kernel<float, float, float><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Layer-0 input: rows 0..T-1 = embeddings of segment s, rows T..T'-1 = the
// memory-token embeddings (appended after the segment).
// ---------------------------------------------------------------------------
template <typename TE>
__global__ void init_first_layer_kernel(const NodeEntry* nodes, int T, int Tp, int d,
                                        const TE* emb, const float* mem_emb, float* h) {
  const NodeEntry nd = nodes[blockIdx.y];
  if (nd.y != 0) return;
  const int t = blockIdx.x;
  float* dst = h + ((long long)nd.z * Tp + t) * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x)
    dst[c] = t < T ? ld(emb, ((long long)nd.x * T + t) * d + c) : mem_emb[(long long)(t - T) * d + c];
}

// Tensor-core path: one block per 32 rows x 64 columns of a layer-0 node.
// Rows are read (and the fp16 copy written) row-major through a shared tile,
// then the fp32 residual is written in the row-blocked layout, where the
// tile's 32 x 64 values form one contiguous run of 2048 floats.
__global__ void init_first_layer_blocked_kernel(const NodeEntry* nodes, int T, int Tp, int d, const bf16* emb,
                                                const float* mem_emb, float* h, f16* xb) {
  grid_dependency_sync();
  __shared__ float tile[32][65];
  const NodeEntry nd = nodes[blockIdx.z];
  if (nd.y != 0) return;
  const int r0 = blockIdx.x * 32, c0 = blockIdx.y * 64;
  for (int e = threadIdx.x; e < 32 * 64; e += blockDim.x) {
    const int r = e >> 6, c = e & 63;
    const int t = r0 + r, col = c0 + c;
    float v = 0.f;
    if (col < d && t < Tp) {
      v = t < T ? __bfloat162float(emb[((long long)nd.x * T + t) * d + col]) : mem_emb[(long long)(t - T) * d + col];
      xb[((long long)nd.z * Tp + t) * d + col] = __float2half_rn(v);
    }
    tile[r][c] = v;
  }
  __syncthreads();
  float* hs = h + (long long)nd.z * rows_blocked(Tp) * d;
  for (int e = threadIdx.x; e < 32 * 64; e += blockDim.x) {
    const int g = e >> 7, r = (e >> 2) & 31, cc = e & 3;   // column group, row, column in group
    const int col = c0 + g * 4 + cc;
    if (col < d) hs[h_blocked_offset(r0 + r, col, d)] = tile[r][g * 4 + cc];
  }
}

cudaError_t launch_init_first_layer(const Dims& dm, const NodeEntry* nodes, int n, int T, int Tp,
                                    const void* emb, const float* mem_emb, float* h, f16* xb, cudaStream_t st) {
  if (dm.bf16) {
    if (!xb || dm.d % 4) return cudaErrorInvalidValue;
    dim3 grid(rows_blocked(Tp) / 32, (dm.d + 63) / 64, n);
    return launch_pdl(init_first_layer_blocked_kernel, grid, dim3(256), 0, st, nodes, T, Tp, dm.d, (const bf16*)emb,
                      mem_emb, h, xb);
  } else {
    dim3 grid(Tp, n);
    init_first_layer_kernel<float><<<grid, 256, 0, st>>>(nodes, T, Tp, dm.d, (const float*)emb, mem_emb, h);
  }
  return cudaGetLastError();
}

// Row sums of squares of the row-blocked residual (tensor-core path) as the
// RMSNorm partials of the QKV epilogue: part 0 holds the whole row's sum, the
// other parts 0 (used for the layer-0 input when no memory read runs first).
// One warp per 32-row block: lane r walks row r's column groups, so the warp
// reads each block's 32 x 4 floats of a group as one contiguous 512 bytes.
__global__ void row_sumsq_kernel(const NodeEntry* nodes, int Tp, int d, const float* h, float* rsq,
                                 long long rsq_slot_stride, int parts, int pitch) {
  grid_dependency_sync();
  const NodeEntry nd = nodes[blockIdx.y];
  const int r = blockIdx.x * 32 + threadIdx.x;
  const float4* hb = reinterpret_cast<const float4*>(h + (long long)nd.z * rows_blocked(Tp) * d +
                                                     (long long)blockIdx.x * 32 * d) + threadIdx.x;
  float ss = 0.f;
  for (int g = 0; g < d / 4; ++g) {
    const float4 v = hb[(long long)g * 32];
    ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
  }
  if (r >= Tp) return;
  float* out = rsq + (long long)nd.z * rsq_slot_stride + r;
  out[0] = ss;
  for (int q = 1; q < parts; ++q) out[(long long)q * pitch] = 0.f;
}

cudaError_t launch_row_sumsq(const Dims& dm, const NodeEntry* nodes, int n, int Tp, const float* h, float* rsq,
                             long long rsq_slot_stride, int parts, int pitch, cudaStream_t st) {
  if (dm.d % 4) return cudaErrorInvalidValue;
  return launch_pdl(row_sumsq_kernel, dim3(rows_blocked(Tp) / 32, n), dim3(32), 0, st, nodes, Tp, dm.d, h, rsq,
                    rsq_slot_stride, parts, pitch);
}

// ---------------------------------------------------------------------------
// RMSNorm (gain folded into the next projection): xb = h * rsqrt(mean h^2 + eps)
// One warp per row.
// ---------------------------------------------------------------------------
template <typename TX>
__global__ void rmsnorm_kernel(const NodeEntry* nodes, int Tp, int row0, int nrows, int d, const float* h, TX* xb,
                               float eps) {
  const NodeEntry nd = nodes[blockIdx.y];
  const int rr = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (rr >= nrows) return;
  const int row = row0 + rr;
  const long long off = ((long long)nd.z * Tp + row) * d;
  const float* src = h + off;
  float ss = 0.f;
  for (int c = lane; c < d; c += 32) ss = fmaf(src[c], src[c], ss);
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)d + eps);
  for (int c = lane; c < d; c += 32) st(xb, off + c, src[c] * r);
}

cudaError_t launch_rmsnorm(const Dims& dm, const NodeEntry* nodes, int n, int Tp, int row0, int nrows,
                           const float* h, void* xb, float eps, cudaStream_t st) {
  dim3 grid((nrows + 7) / 8, n);
  if (dm.bf16) rmsnorm_kernel<f16><<<grid, 256, 0, st>>>(nodes, Tp, row0, nrows, dm.d, h, (f16*)xb, eps);
  else rmsnorm_kernel<float><<<grid, 256, 0, st>>>(nodes, Tp, row0, nrows, dm.d, h, (float*)xb, eps);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Memory read, feature step: phi = DPFP_nu(q) per row, stored as fp32 (fp32
// path) or fp16 (tensor-core path; a value past the fp16 range sets the
// error word), and inv_den = 1 / (z_l . phi + eps) computed from the stored
// (rounded) features so that numerator and denominator see the same phi.
// DPFP: r = [relu(q); relu(-q)], phi[(n-1) 2dk + j] = r_j r_{(j-n) mod 2dk}.
// One warp per row.
// ---------------------------------------------------------------------------
// fp32 value rounded to tf32 (10-bit mantissa, round to nearest, ties away):
// the precision at which the tensor-core read multiplies it.
__device__ __forceinline__ float round_tf32(float v) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(v));
  return __uint_as_float(r);
}

template <bool TF32>
__global__ void dpfp_read_kernel(const NodeEntry* nodes, int Tp, int dk, int nu, int P,
                                 const float* qm, const float* z_state, float* phi, float* inv_den,
                                 float eps) {
  grid_dependency_sync();
  extern __shared__ float r_sh[];   // [8 warps][2 dk]
  const NodeEntry nd = nodes[blockIdx.y];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= Tp) return;
  float* r = r_sh + warp * 2 * dk;
  const long long roff = (long long)nd.z * Tp + row;
  const float* q = qm + roff * dk;
  for (int j = lane; j < dk; j += 32) {
    const float x = q[j];
    r[j] = fmaxf(x, 0.f);
    r[j + dk] = fmaxf(-x, 0.f);
  }
  __syncwarp();
  const int n2 = 2 * dk;
  const float* z = z_state + (long long)nd.y * P;
  float* out = phi + roff * P;
  float dot = 0.f;
  for (int n = 1; n <= nu; ++n) {      // block n: r_j * r_{(j - n) mod 2dk} (nu <= 2 dk)
    for (int j = lane; j < n2; j += 32) {
      const int jj = j - n < 0 ? j - n + n2 : j - n;
      const int p = (n - 1) * n2 + j;
      const float f = TF32 ? round_tf32(r[j] * r[jj]) : r[j] * r[jj];
      out[p] = f;
      dot = fmaf(f, z[p], dot);   // the stored (operand-precision) value
    }
  }
  dot = warp_sum(dot);
  if (lane == 0) inv_den[roff] = 1.f / (dot + eps);
}

// phi [slot][T'][P] fp32; on the tensor-core path (bf16 mode) rounded to tf32,
// the operand precision of the read product.
cudaError_t launch_dpfp_read(const Dims& dm, const NodeEntry* nodes, int n, int Tp, const float* qm,
                             const float* z_state, float* phi, float* inv_den, cudaStream_t st) {
  dim3 grid((Tp + 7) / 8, n);
  const size_t sh = 8 * 2 * dm.dk * sizeof(float);
  if (dm.bf16)
    return launch_pdl(dpfp_read_kernel<true>, grid, dim3(256), sh, st, nodes, Tp, dm.dk, dm.nu, dm.P, qm, z_state,
                      phi, inv_den, dm.mem_eps);
  dpfp_read_kernel<false><<<grid, 256, sh, st>>>(nodes, Tp, dm.dk, dm.nu, dm.P, qm, z_state, phi, inv_den,
                                                 dm.mem_eps);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// RoPE in place on the q and k columns of qkv [T'][Nqkv]: rotate pairs
// (j, j + hd/2) of every head by angle p * theta^(-2j/hd), p = row index.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void rope_kernel(const NodeEntry* nodes, int Tp, int nheads_qk, int hd, int nqkv,
                            T* qkv, const float2* rope, int rope_pitch) {
  const NodeEntry nd = nodes[blockIdx.y];
  const int t = blockIdx.x;
  const int half = hd / 2;
  T* row = qkv + ((long long)nd.z * Tp + t) * nqkv;
  for (int idx = threadIdx.x; idx < nheads_qk * half; idx += blockDim.x) {
    const int hh = idx / half, j = idx - hh * half;
    const int c1 = hh * hd + j, c2 = c1 + half;
    const float x1 = ld(row, c1), x2 = ld(row, c2);
    const float2 a = rope[(long long)j * rope_pitch + t];
    st(row, c1, x1 * a.x - x2 * a.y);
    st(row, c2, x2 * a.x + x1 * a.y);
  }
}

cudaError_t launch_rope(const Dims& dm, const NodeEntry* nodes, int n, int Tp, void* qkv,
                        const float2* rope, int rope_pitch, cudaStream_t st) {
  dim3 grid(Tp, n);
  if (dm.bf16) return cudaErrorInvalidValue;   // the tensor-core path fuses RoPE into the QKV GEMM
  rope_kernel<float><<<grid, 256, 0, st>>>(nodes, Tp, dm.H + dm.KV, dm.hd, dm.nqkv, (float*)qkv, rope,
                                           rope_pitch);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Causal attention, SIMT (fp32 path): one thread per query row, online
// softmax over key tiles staged in shared memory.  Query head h reads kv
// head h / (H / KV).
// ---------------------------------------------------------------------------
template <typename T, int HD>
__global__ void __launch_bounds__(64) attention_simt_kernel(const NodeEntry* nodes, int Tp, int H, int KV,
                                                            int nqkv, const T* qkv, T* out, float scale) {
  constexpr int KT = 32;
  __shared__ float Ks[KT][HD];
  __shared__ float Vs[KT][HD];
  const NodeEntry nd = nodes[blockIdx.z];
  const int h = blockIdx.y, g = h / (H / KV);
  const int q0 = blockIdx.x * 64;
  const int t = q0 + threadIdx.x;
  const T* base = qkv + (long long)nd.z * Tp * nqkv;
  const int kcol = H * HD + g * HD, vcol = (H + KV) * HD + g * HD;
  float q[HD], acc[HD];
  float mx = -INFINITY, sum = 0.f;
  if (t < Tp) {
#pragma unroll
    for (int e = 0; e < HD; ++e) q[e] = ld(base, (size_t)t * nqkv + h * HD + e) * scale;
  }
#pragma unroll
  for (int e = 0; e < HD; ++e) acc[e] = 0.f;
  const int kend = min(Tp, q0 + 64);
  for (int k0 = 0; k0 < kend; k0 += KT) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < KT * HD; idx += 64) {
      const int r = idx / HD, e = idx - r * HD;
      const int u = k0 + r;
      Ks[r][e] = u < Tp ? ld(base, (size_t)u * nqkv + kcol + e) : 0.f;
      Vs[r][e] = u < Tp ? ld(base, (size_t)u * nqkv + vcol + e) : 0.f;
    }
    __syncthreads();
    if (t < Tp) {
      for (int r = 0; r < KT; ++r) {
        const int u = k0 + r;
        if (u > t) break;
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < HD; ++e) s = fmaf(q[e], Ks[r][e], s);
        const float nm = fmaxf(mx, s);
        const float corr = __expf(mx - nm);
        const float p = __expf(s - nm);
        sum = sum * corr + p;
#pragma unroll
        for (int e = 0; e < HD; ++e) acc[e] = fmaf(acc[e], corr, p * Vs[r][e]);
        mx = nm;
      }
    }
  }
  if (t < Tp) {
    T* o = out + ((long long)nd.z * Tp + t) * (H * HD) + h * HD;
    const float inv = 1.f / sum;
#pragma unroll
    for (int e = 0; e < HD; ++e) st(o, e, acc[e] * inv);
  }
}

template <typename T>
static cudaError_t attention_dispatch(const Dims& dm, const NodeEntry* nodes, int n, int Tp,
                                      const void* qkv, void* out, cudaStream_t st) {
  dim3 grid((Tp + 63) / 64, dm.H, n);
  const float scale = 1.f / sqrtf((float)dm.hd);
  const T* q = (const T*)qkv;
  T* o = (T*)out;
  switch (dm.hd) {
    case 16: attention_simt_kernel<T, 16><<<grid, 64, 0, st>>>(nodes, Tp, dm.H, dm.KV, dm.nqkv, q, o, scale); break;
    case 32: attention_simt_kernel<T, 32><<<grid, 64, 0, st>>>(nodes, Tp, dm.H, dm.KV, dm.nqkv, q, o, scale); break;
    case 64: attention_simt_kernel<T, 64><<<grid, 64, 0, st>>>(nodes, Tp, dm.H, dm.KV, dm.nqkv, q, o, scale); break;
    case 128: attention_simt_kernel<T, 128><<<grid, 64, 0, st>>>(nodes, Tp, dm.H, dm.KV, dm.nqkv, q, o, scale); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_attention_simt(const Dims& dm, const NodeEntry* nodes, int n, int Tp,
                                  const void* qkv, void* out, cudaStream_t st) {
  if (dm.bf16) return cudaErrorInvalidValue;   // the tensor-core path has its own attention kernel
  return attention_dispatch<float>(dm, nodes, n, Tp, qkv, out, st);
}

// ---------------------------------------------------------------------------
// SwiGLU: u = silu(gate) * up, gate = gu[:, 0:F], up = gu[:, F:2F].
// ---------------------------------------------------------------------------
template <typename T>
__global__ void swiglu_kernel(const NodeEntry* nodes, int Tp, int F, const T* gu, T* u) {
  const NodeEntry nd = nodes[blockIdx.y];
  const long long rows = Tp;
  const long long total = rows * F;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long t = i / F, f = i - t * F;
    const T* src = gu + ((long long)nd.z * Tp + t) * 2 * F;
    const float g = ld(src, f), up = ld(src, F + f);
    st(u, ((long long)nd.z * Tp + t) * F + f, g / (1.f + __expf(-g)) * up);
  }
}

cudaError_t launch_swiglu(const Dims& dm, const NodeEntry* nodes, int n, int Tp, const void* gu,
                          void* u, cudaStream_t st) {
  dim3 grid(256, n);
  if (dm.bf16) return cudaErrorInvalidValue;   // fused into the gate/up GEMM on the tensor-core path
  swiglu_kernel<float><<<grid, 256, 0, st>>>(nodes, Tp, dm.F, (const float*)gu, (float*)u);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Layer-pipeline hand-off: the residual rows [Tp][d] (fp32, row-major) after
// the previous stage's last layer are loaded into the slot of this stage's
// first-layer node, and those of this stage's last-layer node are stored.
// Tensor-core path: the residual is row-blocked and the first layer's GEMMs
// read its fp16 copy, which the load writes as the down-projection epilogue
// would have (round to nearest); one block per 32 rows x 64 columns through a
// shared tile, as for the layer-0 input.  fp32 path: row-major copies.
// ---------------------------------------------------------------------------
__global__ void stage_rows_in_blocked_kernel(const NodeEntry* nodes, int layer, int Tp, int d, const float* in,
                                             float* h, f16* xb) {
  __shared__ float tile[32][65];
  const NodeEntry nd = nodes[blockIdx.z];
  if (nd.y != layer) return;
  const int r0 = blockIdx.x * 32, c0 = blockIdx.y * 64;
  for (int e = threadIdx.x; e < 32 * 64; e += blockDim.x) {
    const int r = e >> 6, c = e & 63;
    const int t = r0 + r, col = c0 + c;
    float v = 0.f;
    if (col < d && t < Tp) {
      v = in[(long long)t * d + col];
      xb[((long long)nd.z * Tp + t) * d + col] = __float2half_rn(v);
    }
    tile[r][c] = v;
  }
  __syncthreads();
  float* hs = h + (long long)nd.z * rows_blocked(Tp) * d;
  for (int e = threadIdx.x; e < 32 * 64; e += blockDim.x) {
    const int g = e >> 7, r = (e >> 2) & 31, cc = e & 3;   // column group, row, column in group
    const int col = c0 + g * 4 + cc;
    if (col < d) hs[h_blocked_offset(r0 + r, col, d)] = tile[r][g * 4 + cc];
  }
}

__global__ void stage_rows_out_blocked_kernel(const NodeEntry* nodes, int layer, int Tp, int d, const float* h,
                                              float* out) {
  __shared__ float tile[32][65];
  const NodeEntry nd = nodes[blockIdx.z];
  if (nd.y != layer) return;
  const int r0 = blockIdx.x * 32, c0 = blockIdx.y * 64;
  const float* hs = h + (long long)nd.z * rows_blocked(Tp) * d;
  for (int e = threadIdx.x; e < 32 * 64; e += blockDim.x) {
    const int g = e >> 7, r = (e >> 2) & 31, cc = e & 3;
    const int col = c0 + g * 4 + cc;
    tile[r][g * 4 + cc] = col < d ? hs[h_blocked_offset(r0 + r, col, d)] : 0.f;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < 32 * 64; e += blockDim.x) {
    const int r = e >> 6, c = e & 63;
    const int t = r0 + r, col = c0 + c;
    if (col < d && t < Tp) out[(long long)t * d + col] = tile[r][c];
  }
}

// fp32 path: rows of the node's row-major slot <-> [Tp][d] (to_slot selects the direction)
__global__ void stage_rows_copy_kernel(const NodeEntry* nodes, int layer, int Tp, int d, const float* src,
                                       float* dst, int to_slot) {
  const NodeEntry nd = nodes[blockIdx.y];
  if (nd.y != layer) return;
  const int t = blockIdx.x;
  const long long slot_row = ((long long)nd.z * Tp + t) * d, flat_row = (long long)t * d;
  const float* s = src + (to_slot ? flat_row : slot_row);
  float* o = dst + (to_slot ? slot_row : flat_row);
  for (int c = threadIdx.x; c < d; c += blockDim.x) o[c] = s[c];
}

cudaError_t launch_stage_rows_in(const Dims& dm, const NodeEntry* nodes, int n, int layer, int Tp, const float* in,
                                 float* h, void* xb, cudaStream_t st) {
  if (dm.bf16) {
    if (!xb || dm.d % 4) return cudaErrorInvalidValue;
    dim3 grid(rows_blocked(Tp) / 32, (dm.d + 63) / 64, n);
    stage_rows_in_blocked_kernel<<<grid, 256, 0, st>>>(nodes, layer, Tp, dm.d, in, h, (f16*)xb);
  } else {
    dim3 grid(Tp, n);
    stage_rows_copy_kernel<<<grid, 256, 0, st>>>(nodes, layer, Tp, dm.d, in, h, 1);
  }
  return cudaGetLastError();
}

cudaError_t launch_stage_rows_out(const Dims& dm, const NodeEntry* nodes, int n, int layer, int Tp, const float* h,
                                  float* out, cudaStream_t st) {
  if (dm.bf16) {
    if (dm.d % 4) return cudaErrorInvalidValue;
    dim3 grid(rows_blocked(Tp) / 32, (dm.d + 63) / 64, n);
    stage_rows_out_blocked_kernel<<<grid, 256, 0, st>>>(nodes, layer, Tp, dm.d, h, out);
  } else {
    dim3 grid(Tp, n);
    stage_rows_copy_kernel<<<grid, 256, 0, st>>>(nodes, layer, Tp, dm.d, h, out, 0);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Final hidden states: node (s, L-1) writes rows 0..T-1 of its residual
// stream to out[s*T + t].
// ---------------------------------------------------------------------------
template <typename TO>
__global__ void output_kernel(const NodeEntry* nodes, int T, int Tp, int d, int last, const float* h, TO* out) {
  const NodeEntry nd = nodes[blockIdx.y];
  if (nd.y != last) return;
  const int t = blockIdx.x;
  const float* src = h + ((long long)nd.z * Tp + t) * d;
  const long long o = ((long long)nd.x * T + t) * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) st(out, o + c, src[c]);
}

cudaError_t launch_output(const Dims& dm, const NodeEntry* nodes, int n, int T, int Tp,
                          const float* h, void* out, cudaStream_t st) {
  dim3 grid(T, n);
  if (dm.bf16) output_kernel<bf16><<<grid, 256, 0, st>>>(nodes, T, Tp, dm.d, dm.L - 1, h, (bf16*)out);
  else output_kernel<float><<<grid, 256, 0, st>>>(nodes, T, Tp, dm.d, dm.L - 1, h, (float*)out);
  return cudaGetLastError();
}

// fp32 -> bf16 (round to nearest even) -> fp16 container
__global__ void convert_bf16_as_f16_kernel(const float* src, f16* dst, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = __float2half_rn(__bfloat162float(__float2bfloat16_rn(src[i])));
}

// fp32 -> fp16 (round to nearest even)
__global__ void convert_f16_kernel(const float* src, f16* dst, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = __float2half_rn(src[i]);
}

cudaError_t launch_convert(const float* src, void* dst, size_t n, int mode, cudaStream_t st) {
  if (mode == CONVERT_COPY_F32) return cudaMemcpyAsync(dst, src, n * sizeof(float), cudaMemcpyDeviceToDevice, st);
  if (mode == CONVERT_F16) convert_f16_kernel<<<1184, 256, 0, st>>>(src, (f16*)dst, n);
  else convert_bf16_as_f16_kernel<<<1184, 256, 0, st>>>(src, (f16*)dst, n);
  return cudaGetLastError();
}

}  // namespace armt
