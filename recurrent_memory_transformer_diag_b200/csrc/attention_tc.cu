// Batched causal attention on the 5th-generation tensor cores (tcgen05,
// TMEM accumulators, TMA-fed operands), head_dim 64 or 128.
//
// The wave's nodes are a batch: a CTA handles one 128-row query tile of one
// node for the H/KV query heads that share a kv head, so the node's keys and
// values for that kv head stream through one CTA (Pith review of arXiv
// 2506.05229, Figure 5: diagonal batching treats the groups as a batch for
// attention).  Each node attends only over the T' rows of its own segment
// plus memory tokens, causally.
//
// Two softmax warpgroups (A: warps 4..7, B: warps 8..11; one thread per query
// row) take the even and the odd query heads of the group, so two heads are
// in flight and share every K/V tile; each has its own MMA-issuer warp (1 for
// A, 2 for B) in the control warpgroup (warp 0 TMA, warp 3 idle), which hands
// most of its registers to the softmax warpgroups (setmaxnreg: 232 registers
// per softmax thread, 40 per control thread; with 168 each, the softmax
// spilled and ran 7.5 % slower).  Per key tile j and warpgroup w:
//   MMA  S_w = Q_w K_j^T          (M=128 queries, N=128 keys, K=hd) -> TMEM
//   softmax: row max, p = exp2(s - m) and its fp32 row sum in registers; P_w
//            (fp16 pairs) written to TMEM
//   MMA  O_w += P_w V_j           (M=128, N=hd, K=128 keys; P_w read from
//        TMEM), O_w stays in TMEM
// The running max m is only raised when a row's max grows by more than 8 (in
// log2 units): then that row of O_w and its row sum are rescaled; otherwise
// the stale max is kept (p <= 2^8 fits fp16 and the row sum uses the same
// max, so the result is exact).  V is read as V^T (written transposed by the
// QKV epilogue): every shared-memory operand is K-major.
//
// TMEM (512 columns).  hd = 64: S_A, S_B (128 each), O_A, O_B (64 each), P_A,
// P_B (64 each); S(j+1) is issued before O(j), as soon as the softmax holds
// the scores of step j in registers.  hd = 128: S_A, S_B, O_A, O_B take 128
// columns each and P_w is written over the first 64 columns of S_w (the
// scores are in registers by then), so S(j+1) is issued after O(j) (MMAs of
// one issuing thread run in order) and the other warpgroup's products fill
// the tensor core meanwhile.  Shared memory at hd = 128: one Q buffer per
// warpgroup, three K and two V stages (224 KB).
//
// All mbarrier waits are bounded; on timeout the kernel sets the error word,
// drains its copies and MMAs, frees TMEM and exits.
#include "armt_internal.cuh"
#include "tcgen05_ptx.cuh"

namespace armt {

namespace {

using namespace tc;

constexpr int BQ = 128;                 // query rows per tile
constexpr int BKEY = 128;               // keys per tile
// Warpgroup 0: warp 0 TMA, warps 1 / 2 MMA issue for softmax warpgroup A / B,
// warp 3 idle; warpgroups 1 and 2 (warps 4..7, 8..11): softmax A and B.  The
// control warpgroup gives registers to the softmax ones (setmaxnreg): of the
// 384 x 168 registers the block is launched with, 128 x 40 + 256 x 232; on
// each SM sub-partition (one control and two softmax warps) 40 + 2 x 232 = 3 x 168.
constexpr int NUM_THREADS = 384;
constexpr int CTRL_REGS = 40, SOFTMAX_REGS = 232;
static_assert(128 * CTRL_REGS + 256 * SOFTMAX_REGS <= NUM_THREADS * 168, "register split");
constexpr int HALF_BYTES = 128 * 128;   // 128 rows x 64 dims (fp16): one 128-byte-swizzled operand block
constexpr int TMEM_COLS = 512;

// Tile geometry per head_dim.  A Q or K tile is hd / 64 blocks of 128 rows x
// 64 dims (a 128-byte swizzle row holds 64 fp16 values); a V^T stage is two
// blocks of hd rows (dims) x 64 keys.
template <int HD_>
struct AttnShape {
  static constexpr int HD = HD_;
  static constexpr int Q_BYTES = BQ * HD * 2;          // 16 / 32 KB
  static constexpr int K_BYTES = BKEY * HD * 2;        // 16 / 32 KB
  static constexpr int VT_BLK = HD * 128;              // hd rows of 64 keys
  static constexpr int VT_BYTES = 2 * VT_BLK;          // one 128-key stage
  static constexpr int QB = HD == 64 ? 2 : 1;          // Q buffers per warpgroup (2: next head loaded ahead)
  static constexpr int K_STAGES = HD == 64 ? 4 : 3;    // K is needed first (S of the next step): deeper ring
  static constexpr int V_STAGES = HD == 64 ? 3 : 2;    // V^T only at O, a softmax later
  static constexpr bool P_IN_S = HD == 128;            // P written over S (TMEM holds 2 S + 2 O of 128 columns)
  static constexpr int OFF_Q = 0;                                // [2 warpgroups][QB buffers]
  static constexpr int OFF_K = OFF_Q + 2 * QB * Q_BYTES;         // [K_STAGES]
  static constexpr int OFF_VT = OFF_K + K_STAGES * K_BYTES;      // [V_STAGES][2 blocks of VT_BLK]
  static constexpr int OFF_BAR = OFF_VT + V_STAGES * VT_BYTES;
  static constexpr int SMEM_TOTAL = OFF_BAR + 512 + 1024;
  static_assert(SMEM_TOTAL <= 227 * 1024, "shared memory");
  // TMEM columns: S_A, S_B (fp32 scores, 128 each), O_A, O_B (fp32, hd each),
  // P_A, P_B (fp16 probabilities packed in pairs, 64 each; over S at hd = 128)
  static constexpr int TM_S = 0, TM_O = 2 * BKEY;
  static constexpr int TM_P = P_IN_S ? TM_S : TM_O + 2 * HD;
  static constexpr int TM_P_STRIDE = P_IN_S ? BKEY : BKEY / 2;
  static_assert(TM_O + 2 * HD <= TMEM_COLS && TM_P + 2 * TM_P_STRIDE <= TMEM_COLS, "tensor memory");
};
constexpr float RESCALE_THRESHOLD = 8.f;
// Share of the exponentials taken off the MUFU unit (every POLY_EVERY-th
// pair by polynomial; 0 = none).  An eighth measured fastest on the 1B wave,
// about 3 % ahead of none and 5 % ahead of a quarter (the softmax is mostly
// issue-bound, so a larger share costs more FMA issue than it saves).
constexpr int POLY_EVERY = 8;

struct AttnParams {
  const NodeEntry* nodes;
  int n_nodes;
  int Tp;            // rows per node
  int H, KV, nqkv;
  int q_tiles;
  float scale_log2;  // log2(e) / sqrt(hd)
  f16* out;          // [slot][Tp][H*hd]
  unsigned* err;
};

// 2^x by the hardware approximation (PTX ex2.approx.ftz.f32; 2^-inf = +0).
// Its relative error is far below the fp16 rounding that P goes through next.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// A packed pair of fp32 (sm_100a's f32x2 FMA: two lanes per instruction) and
// the three-input max.  (Packed row sums cost more in register pairing than
// they save.)
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x on the FMA pipe, for the share of the probabilities that bypasses the
// MUFU unit: x = j + f with j = round(x) (the 1.5 * 2^23 shift puts j in the
// low mantissa bits of t) and f in [-1/2, 1/2]; 2^f by a degree-3 polynomial
// fitted here by the Remez exchange for minimal relative error (7.5e-5, well
// under the fp16 rounding P goes through next); 2^j is added to the exponent
// field.  x is clamped to -125 so the exponent field stays normal (-inf ->
// 2^-125, zero in fp16).
__device__ __forceinline__ float ex2_poly(float x) {
  x = fmaxf(x, -125.f);
  const float t = x + 12582912.f;
  const float f = x - (t - 12582912.f);
  float q = fmaf(0.0551716685f, f, 0.2426111251f);
  q = fmaf(q, f, 0.6932609677f);
  q = fmaf(q, f, 0.9999280572f);
  // bits(t) = bits(1.5 * 2^23) + j and bits(1.5 * 2^23) << 23 == 0 (mod 2^32)
  return __uint_as_float(__float_as_uint(q) + (__float_as_uint(t) << 23));
}

template <int HD_>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tm_qk, const __grid_constant__ CUtensorMap tm_vt,
                        const AttnParams p) {
  using SH = AttnShape<HD_>;
  constexpr int HD = SH::HD, QB = SH::QB, K_STAGES = SH::K_STAGES, V_STAGES = SH::V_STAGES;
  constexpr int Q_BYTES = SH::Q_BYTES, K_BYTES = SH::K_BYTES, VT_BLK = SH::VT_BLK, VT_BYTES = SH::VT_BYTES;
  constexpr int OFF_Q = SH::OFF_Q, OFF_K = SH::OFF_K, OFF_VT = SH::OFF_VT, OFF_BAR = SH::OFF_BAR;
  constexpr int TM_S = SH::TM_S, TM_O = SH::TM_O, TM_P = SH::TM_P, TM_P_STRIDE = SH::TM_P_STRIDE;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bar;                        // [w][2]
  uint64_t* q_empty = q_full + 4;                // [w][2]
  uint64_t* k_full = q_empty + 4;                // [K_STAGES]
  uint64_t* k_empty = k_full + K_STAGES;         // [K_STAGES]
  uint64_t* v_full = k_empty + K_STAGES;         // [V_STAGES]
  uint64_t* v_empty = v_full + V_STAGES;         // [V_STAGES]
  uint64_t* s_full = v_empty + V_STAGES;         // [w]
  uint64_t* s_empty = s_full + 2;                // [w]
  uint64_t* p_full = s_empty + 2;                // [w]
  uint64_t* o_full = p_full + 2;                 // [w]
  uint64_t* drain = o_full + 2;                  // [w]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  grid_dependency_sync();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // an earlier kernel of this forward already gave up on a wait: do nothing
  // (one thread reads the word, so the whole CTA takes the same decision)
  __shared__ unsigned skip_cta;
  if (threadIdx.x == 0) skip_cta = *reinterpret_cast<volatile unsigned*>(p.err) & ERR_WAIT_TIMEOUT_MASK;
  __syncthreads();
  if (skip_cta) return;
  const int grp = p.H / p.KV;                       // query heads per kv head
  const int heads_a = (grp + 1) / 2, heads_b = grp / 2;   // warpgroup A: even heads, B: odd heads
  const int per_qt = p.n_nodes * p.KV;
  const int n_items = per_qt * p.q_tiles;
  // work item u: longest query tiles first, then node, then kv head
  auto decode = [&](int u, NodeEntry& nd, int& g, int& q0, int& ntiles) {
    const int qt = p.q_tiles - 1 - u / per_qt;
    const int rem = u - (u / per_qt) * per_qt;
    nd = p.nodes[rem / p.KV];
    g = rem - (rem / p.KV) * p.KV;
    q0 = qt * BQ;
    ntiles = (min(p.Tp, q0 + BQ) + BKEY - 1) / BKEY;   // key tiles 0..qt
  };

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2 * QB; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_empty[b], 1);
    }
    for (int b = 0; b < K_STAGES; ++b) {
      mbar_init(&k_full[b], 1);
      mbar_init(&k_empty[b], 2);   // one release per MMA warp
    }
    for (int b = 0; b < V_STAGES; ++b) {
      mbar_init(&v_full[b], 1);
      mbar_init(&v_empty[b], 2);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&s_full[w], 1);
      mbar_init(&s_empty[w], 4);
      mbar_init(&p_full[w], 4);
      mbar_init(&o_full[w], 1);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // The CTA's work is one sequence of steps over its work items item_of(0),
  // item_of(1), ...; within an item, head k (of each warpgroup)
  // and key tile j, step t = k * ntiles + j.  Warpgroup B has no step t when
  // k >= heads_b (odd group size).  kv0 / qh0_* / sw0_* count the K/V tiles,
  // heads and steps of each warpgroup consumed by the earlier items, so every
  // barrier phase follows from them.
  // The CTA's r-th work item: rounds of gridDim.x items, each round visited
  // in the opposite direction to the previous one.  Items come heaviest first,
  // so a CTA with a heavier item in one round gets a lighter one in the next
  // (critical-path load on a full 1B wave 40 tile-steps instead of 43 with
  // plain striding; mean 38.9).  >= n_items past the CTA's last item.
  auto item_of = [&](int r) {
    const int G = gridDim.x;
    return r * G + ((r & 1) ? G - 1 - (int)blockIdx.x : (int)blockIdx.x);
  };
  struct Cursor {   // fields per warpgroup spelled out: no dynamically indexed (local-memory) arrays
    int r, u, t, j, k, ntiles, nA, nB, kv0, qh0_a, qh0_b, sw0_a, sw0_b;   // t = k * ntiles + j
  };
  auto load_item = [&](Cursor& c) {
    NodeEntry nd; int g, q0;
    decode(c.u, nd, g, q0, c.ntiles);
    c.nA = heads_a * c.ntiles;
    c.nB = heads_b * c.ntiles;
  };
  auto first_step = [&](Cursor& c) {
    c.r = 0; c.u = item_of(0); c.t = 0; c.j = 0; c.k = 0; c.kv0 = 0; c.qh0_a = c.qh0_b = 0; c.sw0_a = c.sw0_b = 0;
    load_item(c);
  };
  auto advance = [&](Cursor& c) -> bool {
    if (c.t + 1 < c.nA) {
      ++c.t;
      if (++c.j == c.ntiles) { c.j = 0; ++c.k; }
      return true;
    }
    const int u = item_of(c.r + 1);
    if (u >= n_items) return false;
    ++c.r;
    c.kv0 += c.nA;
    c.qh0_a += heads_a;
    c.qh0_b += heads_b;
    c.sw0_a += c.nA;
    c.sw0_b += c.nB;
    c.u = u;
    c.t = 0; c.j = 0; c.k = 0;
    load_item(c);
    return true;
  };

  if (warp < 4) {
  // control warpgroup: hands registers to the softmax warpgroups
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(CTRL_REGS));
  if (warp == 0) {
    {
      // ---------------- TMA producer (the whole warp runs the loop; one elected lane issues) ----------------
      const bool issuer = elect_one();
      // Per step: K_t (3-stage ring), then V^T of the previous step (2-stage
      // ring), so K runs about two steps ahead of the tensor core and V one.
      // Q tiles (two buffers per warpgroup) are loaded when a head is about to
      // start at the latest, and one head ahead whenever the buffer is free.
      bool ok = true;
      uint32_t armed = 0;   // bits 0-3: Q buffers, 4-6: K stages, 8-9: V stages with loads in flight
      int qi_a = 0, qi_b = 0;            // Q loads issued per warpgroup
      int qr_a = 0, qk_a = 0;   // item round and head of warpgroup A's next Q load
      int qr_b = 0, qk_b = 0;
      // Q load for warpgroup w's next head; block: wait for the buffer, else only if it is free now.
      // Returns 1 issued, 0 buffer busy, -1 wait failed.
      auto q_issue = [&](int w, bool block) -> int {
        int& qi = w ? qi_b : qi_a;
        int& qr = w ? qr_b : qr_a;
        int& qk = w ? qk_b : qk_a;
        const int qb = w * QB + qi % QB;
        const uint32_t par = ((qi / QB) & 1) ^ 1;
        if (block) {
          if (!mbar_wait_warp(&q_empty[qb], par, abort_flag)) return -1;
        } else if (!__any_sync(0xffffffffu, mbar_try_wait(&q_empty[qb], par))) {
          return 0;
        }
        NodeEntry nd; int g, q0, nt;
        decode(item_of(qr), nd, g, q0, nt);
        if (issuer) mbar_expect_tx(&q_full[qb], Q_BYTES);
#pragma unroll
        for (int h = 0; h < HD / 64; ++h)   // 64-dim blocks of the head
          if (issuer)
            tma_load_3d(&tm_qk, &q_full[qb], smem + OFF_Q + qb * Q_BYTES + h * HALF_BYTES,
                        (g * grp + w + 2 * qk) * HD + h * 64, q0, nd.z);
        armed |= 1u << qb;
        ++qi;
        if (++qk >= (w ? heads_b : heads_a)) { qk = 0; ++qr; }
        return 1;
      };
      auto load_v = [&](const Cursor& c) -> bool {
        const int kidx = c.kv0 + c.t, vs = kidx % V_STAGES;
        const int j = c.j;
        if (!mbar_wait_warp(&v_empty[vs], ((kidx / V_STAGES) & 1) ^ 1, abort_flag)) return false;
        NodeEntry nd; int g, q0, nt;
        decode(c.u, nd, g, q0, nt);
        if (issuer) mbar_expect_tx(&v_full[vs], VT_BYTES);
        uint8_t* vt = smem + OFF_VT + vs * VT_BYTES;
        const int vt_outer = nd.z * p.KV + g;
        if (issuer) tma_load_3d(&tm_vt, &v_full[vs], vt, j * BKEY, 0, vt_outer);
        if (issuer) tma_load_3d(&tm_vt, &v_full[vs], vt + VT_BLK, j * BKEY + 64, 0, vt_outer);
        armed |= 256u << vs;
        return true;
      };
      if (blockIdx.x < n_items) {
        Cursor c, prev;
        first_step(c);
        bool has_prev = false;
        while (ok) {
          const int k = c.k, j = c.j;
          // this step's Q tiles must be on their way (normally issued a head earlier)
          const int ha = c.qh0_a + k, hb = c.qh0_b + k;
          while (ok && qi_a <= ha) ok = q_issue(0, true) > 0;
          if (k < heads_b)
            while (ok && qi_b <= hb) ok = q_issue(1, true) > 0;
          if (!ok) break;
          {   // K_t
            const int kidx = c.kv0 + c.t, ks = kidx % K_STAGES;
            if (!mbar_wait_warp(&k_empty[ks], ((kidx / K_STAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
            NodeEntry nd; int g, q0, nt;
            decode(c.u, nd, g, q0, nt);
            if (issuer) mbar_expect_tx(&k_full[ks], K_BYTES);
#pragma unroll
            for (int h = 0; h < HD / 64; ++h)
              if (issuer)
                tma_load_3d(&tm_qk, &k_full[ks], smem + OFF_K + ks * K_BYTES + h * HALF_BYTES, (p.H + g) * HD + h * 64,
                            j * BKEY, nd.z);
            armed |= 16u << ks;
          }
          if (has_prev && !load_v(prev)) { ok = false; break; }
          // one head ahead, if that buffer is already free
          // (B's latest head in this item is min(k, heads_b - 1))
          if (qi_a == ha + 1 && item_of(qr_a) < n_items) q_issue(0, false);
          if (heads_b > 0 && qi_b == c.qh0_b + min(k, heads_b - 1) + 1 && item_of(qr_b) < n_items) q_issue(1, false);
          prev = c;
          has_prev = true;
          if (!advance(c)) break;
        }
        if (ok && has_prev && !load_v(prev)) ok = false;
      }
      if (!ok) {
        if (issuer) atomicOr(p.err, 16u);
        *abort_flag = 1;
      }
      if (*abort_flag) {   // let every issued copy land before the CTA exits
        const unsigned long long t0 = global_ns();
        for (int b = 0; b < 2 * QB; ++b)
          if (armed & (1u << b))
            while (!mbar_try_wait(&q_full[b], 0) && !mbar_try_wait(&q_full[b], 1) && global_ns() - t0 < WAIT_LIMIT_NS) {}
        for (int b = 0; b < K_STAGES; ++b)
          if (armed & (16u << b))
            while (!mbar_try_wait(&k_full[b], 0) && !mbar_try_wait(&k_full[b], 1) && global_ns() - t0 < WAIT_LIMIT_NS) {}
        for (int b = 0; b < V_STAGES; ++b)
          if (armed & (256u << b))
            while (!mbar_try_wait(&v_full[b], 0) && !mbar_try_wait(&v_full[b], 1) && global_ns() - t0 < WAIT_LIMIT_NS) {}
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ---------------- MMA issuers: warp 1 for warpgroup A, warp 2 for B ----------------
    // Each runs the step sequence on the whole warp; one elected lane issues.
    // Two issuers halve the per-step issue chain (waits, descriptors, MMAs);
    // the K/V stages are released by both (count 2).
    const int w = warp - 1;
    const bool issuer = elect_one();
    const uint32_t idesc_s = idesc_f16(BKEY, 0);   // 128 x 128 x 16
    const uint32_t idesc_o = idesc_f16(HD, 0);     // 128 x hd x 16
    auto active = [&](const Cursor& c) { return w == 0 || c.t < c.nB; };
    // S_w = Q_w K_j^T for step c
    auto issue_s = [&](const Cursor& c) -> bool {
      const int hidx = (w ? c.qh0_b : c.qh0_a) + c.k, sidx = (w ? c.sw0_b : c.sw0_a) + c.t, kidx = c.kv0 + c.t;
      const int qb = w * QB + hidx % QB, ks = kidx % K_STAGES;
      if (c.j == 0 && !mbar_wait_warp(&q_full[qb], (hidx / QB) & 1, abort_flag)) return false;
      if (!mbar_wait_warp(&k_full[ks], (kidx / K_STAGES) & 1, abort_flag)) return false;
      if (!mbar_wait_warp(&s_empty[w], (sidx & 1) ^ 1, abort_flag)) return false;
      tc_fence_after();
      const uint32_t qa = smem_u32(smem + OFF_Q + qb * Q_BYTES);
      const uint32_t ka = smem_u32(smem + OFF_K + ks * K_BYTES);
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {   // 16 dims per instruction, 4 per 64-dim block
        const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
        if (issuer) mma_f16(tmem_base + TM_S + w * BKEY, sw128_desc(qa + off), sw128_desc(ka + off), idesc_s, kk > 0);
      }
      if (issuer) mma_commit(&s_full[w]);
      if (c.j == c.ntiles - 1 && issuer) mma_commit(&q_empty[qb]);   // Q buffer free once these MMAs finish
      return true;
    };
    // O_w (+)= P_w [V_j | 1] for step c
    auto issue_o = [&](const Cursor& c) -> bool {
      const int sidx = (w ? c.sw0_b : c.sw0_a) + c.t, kidx = c.kv0 + c.t, vs = kidx % V_STAGES;
      if (!mbar_wait_warp(&p_full[w], sidx & 1, abort_flag)) return false;
      if (!mbar_wait_warp(&v_full[vs], (kidx / V_STAGES) & 1, abort_flag)) return false;
      tc_fence_after();
      const uint32_t pa = tmem_base + TM_P + w * TM_P_STRIDE;   // P_w in TMEM: 8 columns per 16 keys
      const uint32_t va = smem_u32(smem + OFF_VT + vs * VT_BYTES);
#pragma unroll
      for (int kb = 0; kb < BKEY / 64; ++kb)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          if (issuer)
            mma_f16_ts(tmem_base + TM_O + w * HD, pa + (kb * 4 + kk) * 8, sw128_desc(va + kb * VT_BLK + kk * 32),
                       idesc_o, (c.j > 0 || kb > 0 || kk > 0));
      if (issuer) mma_commit(&o_full[w]);
      return true;
    };
    // release of step c's K (V) stage: after this warp's product that reads
    // it, or, for a step warpgroup B does not take, once the stage is loaded
    // (so that the arrival counts toward this use of the stage, not an earlier one)
    auto release_k = [&](const Cursor& c) -> bool {
      const int kidx = c.kv0 + c.t, ks = kidx % K_STAGES;
      if (active(c)) {
        if (issuer) mma_commit(&k_empty[ks]);
      } else {
        if (!mbar_wait_warp(&k_full[ks], (kidx / K_STAGES) & 1, abort_flag)) return false;
        if (issuer) mbar_arrive(&k_empty[ks]);
      }
      return true;
    };
    auto release_v = [&](const Cursor& c) -> bool {
      const int kidx = c.kv0 + c.t, vs = kidx % V_STAGES;
      if (active(c)) {
        if (issuer) mma_commit(&v_empty[vs]);
      } else {
        if (!mbar_wait_warp(&v_full[vs], (kidx / V_STAGES) & 1, abort_flag)) return false;
        if (issuer) mbar_arrive(&v_empty[vs]);
      }
      return true;
    };
    // hd = 64: S of the next step is issued before O of the current one (the
    // S buffer is free once the softmax has the scores in registers), so the
    // softmax finds its next scores computed when it finishes a tile.
    // hd = 128: P_w lives in S_w's columns, so S of the next step follows O of
    // the current one (in issue order, which the tensor core keeps).
    bool ok = true;
    if (blockIdx.x < n_items) {
      Cursor cur;
      first_step(cur);
      if (active(cur)) ok = issue_s(cur);
      if (ok) ok = release_k(cur);
      while (ok) {
        Cursor nxt = cur;
        const bool more = advance(nxt);
        if (SH::P_IN_S) {
          if (active(cur) && !issue_o(cur)) { ok = false; break; }
          if (!release_v(cur)) { ok = false; break; }
        }
        if (more) {
          if (active(nxt) && !issue_s(nxt)) { ok = false; break; }
          if (!release_k(nxt)) { ok = false; break; }
        }
        if (!SH::P_IN_S) {
          if (active(cur) && !issue_o(cur)) { ok = false; break; }
          if (!release_v(cur)) { ok = false; break; }
        }
        if (!more) break;
        cur = nxt;
      }
    }
    if (!ok) {
      if (issuer) atomicOr(p.err, 32u);
      *abort_flag = 1;
    }
    if (issuer) mma_commit(&drain[w]);   // no MMA of this warp still writes TMEM after this arrives
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(&drain[w], 0)) {
      if (global_ns() - t0 > WAIT_LIMIT_NS) break;
    }
  }   // warp 3: nothing to do
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(SOFTMAX_REGS));
    // ---------------- softmax (warpgroup w, one thread per query row) ----------------
    const int w = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int rloc = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_tm = tmem_base + lane_off + TM_S + w * BKEY;
    const uint32_t o_tm = tmem_base + lane_off + TM_O + w * HD;
    const uint32_t p_tm = tmem_base + lane_off + TM_P + w * TM_P_STRIDE;
    const int heads = w == 0 ? heads_a : heads_b;
    int sbase = 0;
    bool ok = true;
    bool first = true;          // no O issued for this warpgroup yet
    bool pend = false;          // a finished head whose O has not been read
    f16* pend_dst = nullptr;    // its output row (nullptr: a padding row)
    float pend_l = 1.f;         // its row sum of P
    int last_sidx = 0;
    // O of a finished head (complete, waited for): normalise by the row sum,
    // fp16 row of the head's hd outputs (64 columns at a time)
    auto finalize = [&](f16* dst, float l) {
#pragma unroll 1
      for (int c = 0; c < HD / 64; ++c) {
        uint32_t orr[64];
        tmem_ld64_nowait(o_tm + c * 64, orr);
        tmem_wait_ld();
        if (dst) {
          const float inv = 1.f / l;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            uint4 v;
            uint32_t* wv = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              __half2 h2 = __floats2half2_rn(__uint_as_float(orr[q * 8 + 2 * i]) * inv,
                                             __uint_as_float(orr[q * 8 + 2 * i + 1]) * inv);
              wv[i] = *reinterpret_cast<uint32_t*>(&h2);
            }
            reinterpret_cast<uint4*>(dst + c * 64)[q] = v;
          }
        }
      }
    };
    for (int r = 0, u = item_of(0); u < n_items && ok; ++r, u = item_of(r)) {
      NodeEntry nd; int g, q0, ntiles;
      decode(u, nd, g, q0, ntiles);
      const int row = q0 + rloc;
      const int nw = heads * ntiles;
      float m_used = -INFINITY;
      float l = 0.f;             // row sum of P at the running max m_used
      for (int t = 0, j = 0, k = 0; t < nw && ok; ++t, j = (j + 1 == ntiles) ? 0 : j + 1, k += (j == 0)) {
        const int sidx = sbase + t;
        if (j == 0) { m_used = -INFINITY; l = 0.f; }
        bool got = mbar_wait(&s_full[w], sidx & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[BKEY];
        tmem_ld64_nowait(s_tm, sr);
        tmem_ld64_nowait(s_tm + 64, sr + 64);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[w]);   // S is in registers: the next S may be computed
        const bool diag = j == ntiles - 1;
        const int k0 = j * BKEY;
        // row max as 8 independent partial maxima (a short dependency chain)
        float m8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
        if (diag) {   // causal mask on the tile that holds the diagonal
#pragma unroll
          for (int i = 0; i < BKEY; i += 2) {
            const float v0 = k0 + i > row ? -INFINITY : __uint_as_float(sr[i]);
            const float v1 = k0 + i + 1 > row ? -INFINITY : __uint_as_float(sr[i + 1]);
            sr[i] = __float_as_uint(v0);
            sr[i + 1] = __float_as_uint(v1);
            m8[(i >> 1) & 7] = max3f(m8[(i >> 1) & 7], v0, v1);
          }
        } else {   // two new values per three-input max
#pragma unroll
          for (int i = 0; i < BKEY; i += 2)
            m8[(i >> 1) & 7] = max3f(m8[(i >> 1) & 7], __uint_as_float(sr[i]), __uint_as_float(sr[i + 1]));
        }
        const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        const float m_tile = mx * p.scale_log2;     // scale > 0: max commutes with it
        float corr = 1.f;
        bool rescale = false;
        if (j == 0) {
          m_used = m_tile;
        } else if (m_tile > m_used + RESCALE_THRESHOLD) {
          corr = exp2f(m_used - m_tile);
          m_used = m_tile;
          rescale = true;
          l *= corr;
        }
        // P = 2^(s - m) as packed fp16 pairs, computed before waiting for the
        // previous O (the exponentials overlap that product)
        // (pairs i with i % POLY_EVERY == POLY_EVERY - 1 on the FMA pipe, the
        // rest on MUFU); row sum in fp32
        // (scale and shift of a pair in one f32x2 FMA); row sum in fp32
        uint32_t pk[BKEY / 2];
        const uint64_t sc2 = f2pack(p.scale_log2, p.scale_log2), nm2 = f2pack(-m_used, -m_used);
        float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < BKEY / 2; ++i) {
          float x0, x1;
          f2unpack(fma_f32x2(f2pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), sc2, nm2), x0, x1);
          const bool poly = POLY_EVERY > 0 && i % (POLY_EVERY > 0 ? POLY_EVERY : 1) == POLY_EVERY - 1;
          const float e0 = poly ? ex2_poly(x0) : ex2_approx(x0);
          const float e1 = poly ? ex2_poly(x1) : ex2_approx(x1);
          l4[i & 3] += e0 + e1;
          const __half2 h2 = __floats2half2_rn(e0, e1);
          pk[i] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
        // the previous step's O must be complete: its MMA read the P buffer,
        // and O is read (head done) or rescaled below
        if (!first) {
          got = mbar_wait(&o_full[w], (sidx - 1) & 1, abort_flag);
          if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
          tc_fence_after();
        }
        tmem_st64(p_tm, pk);        // P_w: this thread's row, keys 2c, 2c+1 in column c
        if (pend) {   // the previous step ended a head: normalise its O and store it
          finalize(pend_dst, pend_l);
          pend = false;
        }
        if (__any_sync(0xffffffffu, rescale)) {   // warp-collective TMEM access; rows that keep their max scale by 1
#pragma unroll 1
          for (int c = 0; c < HD / 64; ++c) {
            uint32_t orr[64];
            tmem_ld64_nowait(o_tm + c * 64, orr);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 64; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * corr);
            tmem_st64(o_tm + c * 64, orr);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[w]);
        first = false;
        if (j == ntiles - 1) {      // head done: its O is read at the next step (or after the last)
          pend = true;
          pend_dst = row < p.Tp ? p.out + ((long long)nd.z * p.Tp + row) * (p.H * HD) + (g * grp + w + 2 * k) * HD
                                : nullptr;
          pend_l = l;
          last_sidx = sidx;
        }
      }
      sbase += nw;
    }
    if (ok && pend) {   // the CTA's last head
      const bool got = mbar_wait(&o_full[w], last_sidx & 1, abort_flag);
      if (__all_sync(0xffffffffu, got)) {
        tc_fence_after();
        finalize(pend_dst, pend_l);
      } else {
        ok = false;
      }
    }
    if (!ok) {
      if (lane == 0) atomicOr(p.err, 64u);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
}

// 3-D tensor map over fp16 [outer][rows][inner], box = box_inner x box_rows,
// rows pitch_rows apart per outer step, 128-byte swizzle, zero fill.
cudaError_t make_map(CUtensorMap* map, const void* base, int inner, int rows, int outer, long long row_pitch_elems,
                     long long outer_pitch_elems, int box_inner, int box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)outer};
  cuuint64_t strides[2] = {(cuuint64_t)row_pitch_elems * 2, (cuuint64_t)outer_pitch_elems * 2};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

bool attention_tc_supported(const Dims& dm) { return dm.bf16 && (dm.hd == 64 || dm.hd == 128); }

int attention_tc_vt_pitch(int Tp) { return (Tp + 7) / 8 * 8; }

cudaError_t setup_attention_tc() {
  if (!get_tensor_map_encoder()) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(attention_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       AttnShape<64>::SMEM_TOTAL);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attention_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             AttnShape<128>::SMEM_TOTAL);
  return e;
}

cudaError_t launch_attention_tc(const Dims& dm, const NodeEntry* nodes, int n, int Tp, int slots, const void* qkv,
                                const void* vt, void* out, unsigned* err, cudaStream_t st) {
  if (!attention_tc_supported(dm)) return cudaErrorInvalidValue;
  CUtensorMap tm_qk, tm_vt;
  const int HD = dm.hd;
  // Q and K tiles: [slot][Tp][nqkv], box 64 dims x 128 rows (hd / 64 boxes per tile)
  cudaError_t e = make_map(&tm_qk, qkv, dm.nqkv, Tp, slots, dm.nqkv, (long long)Tp * dm.nqkv, 64, BQ);
  if (e != cudaSuccess) return e;
  // V^T tiles: [slot * KV + g][hd][pitch], box 64 keys x hd dims
  const int pitch = attention_tc_vt_pitch(Tp);
  e = make_map(&tm_vt, vt, Tp, HD, slots * dm.KV, pitch, (long long)HD * pitch, 64, HD);
  if (e != cudaSuccess) return e;
  AttnParams p;
  p.nodes = nodes;
  p.n_nodes = n;
  p.Tp = Tp;
  p.H = dm.H;
  p.KV = dm.KV;
  p.nqkv = dm.nqkv;
  p.q_tiles = (Tp + BQ - 1) / BQ;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  p.out = (f16*)out;
  p.err = err;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int items = n * dm.KV * p.q_tiles;
  const dim3 grid(items < sms ? items : sms);
  if (HD == 128)
    return launch_pdl(attention_tc_kernel<128>, grid, dim3(NUM_THREADS), AttnShape<128>::SMEM_TOTAL, st, tm_qk,
                      tm_vt, p);
  return launch_pdl(attention_tc_kernel<64>, grid, dim3(NUM_THREADS), AttnShape<64>::SMEM_TOTAL, st, tm_qk, tm_vt,
                    p);
}

}  // namespace armt
