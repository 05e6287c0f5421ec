// Batched causal attention over the nodes of a wave on tensor cores
// (warp-level mma.sync m16n8k16, fp16 operands, fp32 accumulation, online
// softmax).
//
// The wave's nodes are treated as a batch: one CTA per (q tile, query head,
// node), every node attending only over the T' rows of its own segment plus
// memory tokens (Pith review of arXiv 2506.05229, Figure 5: diagonal
// batching treats the groups as a batch for attention).
//
// Per CTA: BM = 16 * WARPS query rows, key/value tiles of 64 rows double
// buffered with cp.async; Q, K, V tiles live in shared memory with a 16-byte
// chunk XOR swizzle (chunk ^ (row & 7)) so ldmatrix reads are conflict free.
// S = Q K^T and O += P V run on mma.sync; P is re-used from the S
// accumulators as the A operand of the second product (register-level reuse,
// no shared-memory round trip).  Query head h reads kv head h / (H / KV).
#include "armt_internal.cuh"

namespace armt {

namespace {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;   // 0 source bytes = zero fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// element offset of (row, 16-byte chunk) in a swizzled [rows][HD] 16-bit tile
template <int HD>
__device__ __forceinline__ int swz(int row, int chunk) {
  return row * HD + ((chunk ^ (row & 7)) << 3);
}

template <int HD, int WARPS>
__global__ void __launch_bounds__(WARPS * 32) attention_mma_kernel(const NodeEntry* nodes, int Tp, int H, int KV,
                                                                   int nqkv, const f16* __restrict__ qkv,
                                                                   f16* __restrict__ out, float scale_log2) {
  constexpr int BM = 16 * WARPS;
  constexpr int BN = 64;
  constexpr int CH = HD / 8;            // 16-byte chunks per row
  constexpr int KS = HD / 16;           // k-steps of S = Q K^T
  constexpr int DT = HD / 8;            // 8-wide dim tiles of O
  constexpr int NT = BN / 8;            // 8-wide key tiles of S
  constexpr int NTHREADS = WARPS * 32;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  f16* sQ = reinterpret_cast<f16*>(smem_raw);
  f16* sK = sQ + BM * HD;              // [2][BN][HD]
  f16* sV = sK + 2 * BN * HD;          // [2][BN][HD]

  const NodeEntry nd = nodes[blockIdx.z];
  const int h = blockIdx.y;
  const int g = h / (H / KV);
  const int qt = gridDim.x - 1 - blockIdx.x;      // longest rows first
  const int q0 = qt * BM;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const f16* base = qkv + (long long)nd.z * Tp * nqkv;
  const f16* Qg = base + h * HD;
  const f16* Kg = base + (H + g) * HD;
  const f16* Vg = base + (H + KV + g) * HD;

  for (int idx = tid; idx < BM * CH; idx += NTHREADS) {
    const int r = idx / CH, c = idx - r * CH;
    const int gr = q0 + r;
    cp_async16(sQ + swz<HD>(r, c), Qg + (long long)min(gr, Tp - 1) * nqkv + c * 8, gr < Tp);
  }
  auto load_kv = [&](int j, int buf) {
    f16* dk = sK + buf * BN * HD;
    f16* dv = sV + buf * BN * HD;
    for (int idx = tid; idx < BN * CH; idx += NTHREADS) {
      const int r = idx / CH, c = idx - r * CH;
      const int gr = j * BN + r;
      const long long off = (long long)min(gr, Tp - 1) * nqkv + c * 8;
      cp_async16(dk + swz<HD>(r, c), Kg + off, gr < Tp);
      cp_async16(dv + swz<HD>(r, c), Vg + off, gr < Tp);
    }
  };
  const int kend = min(Tp, q0 + BM);
  const int ntiles = (kend + BN - 1) / BN;
  load_kv(0, 0);
  cp_async_commit();
  cp_async_wait_all();
  __syncthreads();

  // Q fragments of this warp's 16 rows
  uint32_t qf[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int r = warp * 16 + (lane & 15);
    const int c = ks * 2 + (lane >> 4);
    ldsm_x4(smem_addr(sQ + swz<HD>(r, c)), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
  }

  float o[DT][4];
#pragma unroll
  for (int i = 0; i < DT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int qrow0 = q0 + warp * 16 + (lane >> 2);   // this thread's rows: qrow0, qrow0 + 8
  const int warp_last = q0 + warp * 16 + 15;

  for (int j = 0; j < ntiles; ++j) {
    if (j + 1 < ntiles) load_kv(j + 1, (j + 1) & 1);
    cp_async_commit();
    const int k0 = j * BN;
    if (k0 <= warp_last) {
      const f16* cK = sK + (j & 1) * BN * HD;
      const f16* cV = sV + (j & 1) * BN * HD;
      float s[NT][4];
#pragma unroll
      for (int i = 0; i < NT; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int c = ks * 2 + ((lane >> 3) & 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_addr(cK + swz<HD>(key, c)), b0, b1, b2, b3);
          mma16816(s[2 * np], qf[ks], b0, b1);
          mma16816(s[2 * np + 1], qf[ks], b2, b3);
        }
      }
      // scale, causal mask, online softmax (rows qrow0 and qrow0 + 8)
      const bool diag = k0 + BN - 1 > q0 + warp * 16;
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v = s[nt][e] * scale_log2;
          if (diag) {
            const int key = k0 + nt * 8 + 2 * (lane & 3) + (e & 1);
            const int qr = qrow0 + (e >> 1) * 8;
            if (key > qr) v = -INFINITY;
          }
          s[nt][e] = v;
        }
        mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
        mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float c0 = exp2f(m0 - mn0), c1 = exp2f(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        s[nt][0] = exp2f(s[nt][0] - mn0);
        s[nt][1] = exp2f(s[nt][1] - mn0);
        s[nt][2] = exp2f(s[nt][2] - mn1);
        s[nt][3] = exp2f(s[nt][3] - mn1);
        ps0 += s[nt][0] + s[nt][1];
        ps1 += s[nt][2] + s[nt][3];
      }
      l0 = l0 * c0 + ps0;
      l1 = l1 * c1 + ps1;
#pragma unroll
      for (int dt = 0; dt < DT; ++dt) {
        o[dt][0] *= c0; o[dt][1] *= c0;
        o[dt][2] *= c1; o[dt][3] *= c1;
      }
      // O += P V, P taken from the S accumulators as A fragments
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk) {
        uint32_t a[4];
        a[0] = pack_f16(s[2 * kk][0], s[2 * kk][1]);
        a[1] = pack_f16(s[2 * kk][2], s[2 * kk][3]);
        a[2] = pack_f16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        a[3] = pack_f16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int dp = 0; dp < DT / 2; ++dp) {
          const int key = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
          const int c = dp * 2 + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_addr(cV + swz<HD>(key, c)), b0, b1, b2, b3);
          mma16816(o[2 * dp], a, b0, b1);
          mma16816(o[2 * dp + 1], a, b2, b3);
        }
      }
    }
    cp_async_wait_all();
    __syncthreads();
  }

  // normalise and write: stage the warp's 16 rows in its own part of sQ
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = 1.f / l0, inv1 = 1.f / l1;
  const int r0 = warp * 16 + (lane >> 2);
#pragma unroll
  for (int dt = 0; dt < DT; ++dt) {
    const int col = dt * 8 + 2 * (lane & 3);
    const int c = col >> 3, w = col & 7;
    *reinterpret_cast<uint32_t*>(sQ + swz<HD>(r0, c) + w) = pack_f16(o[dt][0] * inv0, o[dt][1] * inv0);
    *reinterpret_cast<uint32_t*>(sQ + swz<HD>(r0 + 8, c) + w) = pack_f16(o[dt][2] * inv1, o[dt][3] * inv1);
  }
  __syncwarp();
  f16* og = out + ((long long)nd.z * Tp) * (H * HD) + h * HD;
  for (int idx = lane; idx < 16 * CH; idx += 32) {
    const int r = idx / CH, c = idx - r * CH;
    const int row = warp * 16 + r;
    const int gr = q0 + row;
    if (gr < Tp)
      *reinterpret_cast<uint4*>(og + (long long)gr * (H * HD) + c * 8) =
          *reinterpret_cast<const uint4*>(sQ + swz<HD>(row, c));
  }
}

template <int HD, int WARPS>
cudaError_t launch_hd(const Dims& dm, const NodeEntry* nodes, int n, int Tp, const void* qkv, void* out,
                      cudaStream_t st) {
  constexpr int BM = 16 * WARPS;
  const size_t smem = (size_t)(BM * HD + 4 * 64 * HD) * sizeof(f16);
  dim3 grid((Tp + BM - 1) / BM, dm.H, n);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  attention_mma_kernel<HD, WARPS><<<grid, WARPS * 32, smem, st>>>(nodes, Tp, dm.H, dm.KV, dm.nqkv,
                                                                  (const f16*)qkv, (f16*)out, scale_log2);
  return cudaGetLastError();
}

}  // namespace

bool attention_mma_supported(const Dims& dm) { return dm.bf16 && (dm.hd == 64 || dm.hd == 128); }

cudaError_t setup_attention_mma() {
  cudaError_t e = cudaFuncSetAttribute(attention_mma_kernel<64, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (128 * 64 + 4 * 64 * 64) * 2);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attention_mma_kernel<128, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (64 * 128 + 4 * 64 * 128) * 2);
  return e;
}

cudaError_t launch_attention_mma(const Dims& dm, const NodeEntry* nodes, int n, int Tp, const void* qkv, void* out,
                                 cudaStream_t st) {
  if (dm.hd == 64) return launch_hd<64, 8>(dm, nodes, n, Tp, qkv, out, st);
  if (dm.hd == 128) return launch_hd<128, 4>(dm, nodes, n, Tp, qkv, out, st);
  return cudaErrorInvalidValue;
}

}  // namespace armt
