// Paged FP8 decode / MTP-verify grouped-query attention, warp-MMA kernel.
//
// Computes, for every sequence b, KV head h and query row r = (i, g) of the
// head's group (i < q_len new tokens, g < G = Hq/Hkv q-heads per KV head):
//     s_t = sm_scale * k_scale[h] * sum_d q[b,i,h*G+g,d] * code(K[t,h,d])
//     out = v_scale[h] * sum_t softmax(s)_t * code(V[t,h,:]),   t <= L_b - q_len + i
// which is the plain masked SDPA over the dequantised cache with the two
// per-head scales factored out of the dot products.  Sources: the
// FlashAttention-2-style online softmax and the dedicated MQA/GQA kernels of
// the Atlas deep-dive (ainews.cool, "Attention" paragraph), its FP8 with scale
// factors ("Quantisation" paragraph), the fixed-size KV blocks ("Memory
// architecture" paragraph), and the paged FP8 KV cache with MTP K = 4 verify
// of the GB10 page (ainews.surl.tw).
//
// Work split.  CTA (split s, KV head h, sequence b, row block rb) owns the
// KV tokens [s*T, min((s+1)*T, L_b)) and up to 8*NT query rows of the group.
// Each of its 4 warps walks 16-token units (one 16-slot piece of a page)
// round-robin with a private online-softmax state; the warps are combined in
// shared memory at the end.  A sequence with one split writes bf16 output
// directly; otherwise every split writes (O/l, log2-sum-exp) to the workspace
// and the CTA that finishes a (b, h, rb) last -- found with one atomic
// counter, no waiting -- merges the splits and resets the counter.
//
// K/V staging.  Each warp owns a ring of S shared-memory stages; one stage
// holds the K and the V tile of one 16-token unit (16 rows x D bytes each),
// brought in by two 2-D TMA tile loads (cp.async.bulk.tensor, no multicast)
// whose completion is counted on the stage's mbarrier.  The warp keeps S-1
// units in flight while it computes one, without spending registers on
// prefetch.  The tiles land with the 128-byte (D = 128) or 64-byte (D = 64)
// swizzle, which makes every fragment read below bank-conflict-free.
//
// Per unit the warp converts E4M3 -> f16 exactly with cvt.rn.f16x2.e4m3x2 and
// runs both contractions on the tensor cores with mma.sync m16n8k16 (f16 in,
// f32 accumulate), tokens on the M side:
//   S^T[16 tok x 8 rows]  = K_tile[16 x D] . Q^T[D x 8]
//   O^T[D x 8 rows]      += V_tile^T[D x 16] . P^T[16 x 8]
// The head dimension is permuted consistently between K and Q (any
// permutation leaves q.k unchanged) so each thread's K fragment is two
// 16-byte chunks of a token row; for V the thread's 16-byte chunk of one
// token is interleaved with the next token's by byte_perm to form the
// token-pair registers the A operand needs.  P moves from the S^T
// accumulator layout to the PV B-operand layout with one movmatrix.trans.
//
// Every mbarrier wait is bounded (200 ms of wall clock); if one runs out the
// kernel flags ATLAS_DEVERR_TIMEOUT, drains its outstanding loads with the same
// bound and finishes without computing further units.
#include <float.h>
#include <math.h>

#include "atlas_internal.cuh"

namespace atlas {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr uint64_t kWaitLimitNs = 200ull * 1000 * 1000;

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}
__device__ __forceinline__ uint32_t word_of(const uint2& v, int i) { return i == 0 ? v.x : v.y; }

template <int D>
struct Frag;  // one warp-lane's share of a 16-token unit, read from the staged tiles
template <>
struct Frag<128> {
  uint4 k[2][2];  // [token g8 | g8+8][head-dim chunk j]: bytes 64j + 16c .. +16
  uint4 v[4];     // tokens 2c, 2c+1, 2c+8, 2c+9: head dims 16*g8 .. +16
  __device__ __forceinline__ uint32_t kword(int t, int ks) const { return word_of(k[t][ks >> 2], ks & 3); }
  __device__ __forceinline__ uint32_t vword(int q, int w) const { return word_of(v[q], w); }
  __device__ __forceinline__ void zero_v(int q) { v[q] = make_uint4(0, 0, 0, 0); }
  // 128-byte swizzle: 16-byte chunk index XOR (row & 7)
  __device__ __forceinline__ void load(const uint8_t* kt, const uint8_t* vt, int g8, int c) {
    const int ja = g8 & 1;  // odd rows read their chunks in the other order: no bank conflict
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int row = g8 + 8 * t;
      const uint8_t* rb = kt + row * 128;
      const uint4 a = *reinterpret_cast<const uint4*>(rb + ((((4 * ja) + c) ^ (row & 7)) << 4));
      const uint4 b = *reinterpret_cast<const uint4*>(rb + ((((4 * (1 - ja)) + c) ^ (row & 7)) << 4));
      k[t][0] = ja ? b : a;
      k[t][1] = ja ? a : b;
    }
    const int rows[4] = {2 * c, 2 * c + 1, 2 * c + 8, 2 * c + 9};
#pragma unroll
    for (int q = 0; q < 4; ++q)
      v[q] = *reinterpret_cast<const uint4*>(vt + rows[q] * 128 + ((g8 ^ (rows[q] & 7)) << 4));
  }
};
template <>
struct Frag<64> {
  uint4 k[2][1];  // [token g8 | g8+8]: bytes 16c .. +16
  uint2 v[4];     // tokens 2c, 2c+1, 2c+8, 2c+9: head dims 8*g8 .. +8
  __device__ __forceinline__ uint32_t kword(int t, int ks) const { return word_of(k[t][0], ks & 3); }
  __device__ __forceinline__ uint32_t vword(int q, int w) const { return word_of(v[q], w); }
  __device__ __forceinline__ void zero_v(int q) { v[q] = make_uint2(0, 0); }
  // 64-byte swizzle: 16-byte chunk index XOR ((row >> 1) & 3)
  __device__ __forceinline__ void load(const uint8_t* kt, const uint8_t* vt, int g8, int c) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int row = g8 + 8 * t;
      k[t][0] = *reinterpret_cast<const uint4*>(kt + row * 64 + ((c ^ ((row >> 1) & 3)) << 4));
    }
    const int rows[4] = {2 * c, 2 * c + 1, 2 * c + 8, 2 * c + 9};
#pragma unroll
    for (int q = 0; q < 4; ++q)
      v[q] = *reinterpret_cast<const uint2*>(vt + rows[q] * 64 +
                                             ((((g8 >> 1) ^ ((rows[q] >> 1) & 3))) << 4) +
                                             8 * (g8 & 1));
  }
};

// Dynamic shared memory: [ring: warps x S stages x (K tile, V tile)] [mbarriers]
// [page ids]; the warp-combine buffers reuse the ring after the main loop.
struct SmemPlan {
  size_t ring, bars, pids, total;
};
__host__ __device__ inline SmemPlan smem_plan(int D, int S, int split_tokens) {
  SmemPlan sp;
  sp.ring = 0;
  sp.bars = (size_t)kWarps * S * 2 * 16 * D;
  sp.pids = sp.bars + (size_t)kWarps * S * 8;
  sp.total = sp.pids + (size_t)(split_tokens / 16 + 2) * 4 + 1024;  // + alignment slack
  return sp;
}

template <int D, int NT, int S>
__global__ void __launch_bounds__(kThreads, NT == 1 ? 4 : 2)
    paged_decode_mma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV) {
  constexpr int RB = 8 * NT;   // query rows per CTA
  constexpr int NCH = D / 64;  // 16-byte K chunks per token per thread
  constexpr int KS = D / 16;   // k-steps of QK^T
  constexpr int MT = D / 16;   // m-tiles of O^T (head dims)
  constexpr int VB = D / 8;    // V bytes per token per thread
  constexpr int TILE = 16 * D; // bytes of one K (or V) unit tile
  constexpr int STAGE = 2 * TILE;
  static_assert((size_t)kWarps * S * STAGE >= (size_t)(2 * kWarps * RB + kWarps * RB * D) * 4,
                "combine buffers must fit in the ring");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const SmemPlan sp = smem_plan(D, S, p.split_tokens);
  uint8_t* ring = smem + sp.ring;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sp.bars);
  int* s_pid = reinterpret_cast<int*>(smem + sp.pids);
  float* s_m = reinterpret_cast<float*>(ring);  // after the main loop only
  float* s_l = s_m + kWarps * RB;
  float* s_o = s_l + kWarps * RB;
  __shared__ int s_is_last;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, c = lane & 3;
  const int rb = blockIdx.x % p.row_blocks;
  const int split = blockIdx.x / p.row_blocks;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int L = __ldg(p.seq_lens + b);
  const int Rtot = p.q_len * p.G;
  const int row0 = rb * RB;
  const int rows_here = min(RB, Rtot - row0);

  // ---- invalid sequence (shorter than q_len, longer than its block-table row
  // or than the host's max_seq_len): zero this CTA's rows once and flag it
  if (L < p.q_len || L > p.max_blocks * p.ps || L > p.num_splits * p.split_tokens) {
    if (split == 0) {
      if (tid == 0) atomicOr(p.err, ATLAS_DEVERR_SEQ_LEN);
      for (int idx = tid; idx < rows_here * D; idx += kThreads) {
        const int r = row0 + idx / D, d = idx % D;
        const int i = r / p.G, hq = h * p.G + r % p.G;
        p.out[(((size_t)b * p.q_len + i) * p.Hq + hq) * D + d] = __float2bfloat16_rn(0.f);
      }
    }
    return;
  }
  const int t_begin = split * p.split_tokens;
  if (t_begin >= L) return;
  const int t_end = min(t_begin + p.split_tokens, L);
  const int n_split_b = (L + p.split_tokens - 1) / p.split_tokens;

  // ---- page ids of this split (A2: block-table gather), checked once
  const int pg_begin = t_begin / p.ps;
  const int pg_last = (t_end - 1) / p.ps;
  for (int i = tid; i <= pg_last - pg_begin; i += kThreads) {
    int pid = __ldg(p.block_table + (size_t)b * p.max_blocks + pg_begin + i);
    if (pid < 0 || pid >= p.num_pages) {
      atomicOr(p.err, ATLAS_DEVERR_PAGE_ID);
      pid = -1;
    }
    s_pid[i] = pid;
  }
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < S; ++s) mbar_init(&bars[warp * S + s], 1);
    fence_mbar_init();
  }

  // ---- Q fragments (B operand of S^T = K Q^T), bf16 -> f16 (exact in range)
  // k-step ks uses head dims j*64 + 16c + 4w + {0,1 | 2,3}, j = ks/4, w = ks%4.
  uint32_t qf[NT][KS][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int r = row0 + 8 * nt + g8;
    if (r < Rtot) {
      const int i = r / p.G, hq = h * p.G + r % p.G;
      const __nv_bfloat16* qrow = p.q + (((size_t)b * p.q_len + i) * p.Hq + hq) * D;
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        const uint4* src = reinterpret_cast<const uint4*>(qrow + j * 64 + 16 * c);
        const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
        const uint32_t wv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float d0 = __uint_as_float(wv[2 * w] << 16);
          const float d1 = __uint_as_float(wv[2 * w] & 0xFFFF0000u);
          const float d2 = __uint_as_float(wv[2 * w + 1] << 16);
          const float d3 = __uint_as_float(wv[2 * w + 1] & 0xFFFF0000u);
          qf[nt][4 * j + w][0] = pack_f16x2(d0, d1);
          qf[nt][4 * j + w][1] = pack_f16x2(d2, d3);
        }
      }
    } else {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) qf[nt][ks][0] = qf[nt][ks][1] = 0u;
    }
  }

  // ---- causal limits of this thread's accumulator rows (8nt + 2c + e)
  int lim[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int r = row0 + 8 * nt + 2 * c + e;
      lim[nt][e] = (r < Rtot) ? (L - p.q_len + r / p.G) : (L - 1);
    }
  const int min_lim = L - p.q_len + row0 / p.G;
  const float scale2 = __ldg(p.k_scale + h) * p.qk_scale_log2;

  float m_run[NT][2], l_run[NT][2];
  float acc[MT][NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_run[nt][0] = l_run[nt][1] = 0.f;
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;

  __syncthreads();  // page ids and barrier init visible

  // this warp's units: u = warp + kWarps * i, i < n_my
  const int n_units = (t_end - t_begin + 15) / 16;
  const int n_my = (warp < n_units) ? (n_units - warp + kWarps - 1) / kWarps : 0;

  auto unit_t0 = [&](int i) { return t_begin + 16 * (warp + kWarps * i); };
  auto issue = [&](int i) {  // lane 0 only: stage i % S <- unit i
    const int t0 = unit_t0(i);
    uint64_t* bar = &bars[warp * S + i % S];
    const int pid = s_pid[t0 / p.ps - pg_begin];
    if (pid < 0) {  // bad page id: complete the phase with no data
      mbar_arrive(bar);
      return;
    }
    const int row = (pid * p.Hkv + h) * p.ps + (t0 % p.ps);
    uint8_t* dst = ring + (size_t)(warp * S + i % S) * STAGE;
    mbar_arrive_expect_tx(bar, STAGE);
    tma_load_2d(dst, &tmK, 0, row, bar);
    tma_load_2d(dst + TILE, &tmV, 0, row, bar);
  };

  auto compute_unit = [&](int t0, Frag<D>& x) {
    // S^T = K . Q^T  (A3 dequant-to-f16 + A4), two accumulation chains
    float sacc[2][NT][4];
#pragma unroll
    for (int ch = 0; ch < 2; ++ch)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) sacc[ch][nt][0] = sacc[ch][nt][1] = sacc[ch][nt][2] = sacc[ch][nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t a0, a1, a2, a3;
      e4m3x4_to_f16x2x2(x.kword(0, ks), a0, a2);
      e4m3x4_to_f16x2x2(x.kword(1, ks), a1, a3);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        mma_16816(sacc[ks & 1][nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
    }
    float sc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] = (sacc[0][nt][e] + sacc[1][nt][e]) * scale2;

    // causal / tail mask (A5)
    if (t0 + 15 > min_lim) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tok = t0 + g8 + ((e & 2) ? 8 : 0);
          if (tok > lim[nt][e & 1]) sc[nt][e] = -INFINITY;
        }
    }
    if (t0 + 16 > L) {  // tail of the last page: no V garbage may reach P*V
      if (t0 + 2 * c >= L) x.zero_v(0);
      if (t0 + 2 * c + 1 >= L) x.zero_v(1);
      if (t0 + 2 * c + 8 >= L) x.zero_v(2);
      if (t0 + 2 * c + 9 >= L) x.zero_v(3);
    }

    // online softmax (A6): row max over the 16 tokens, rescale, P
    uint32_t pb[NT][2];
    bool changed = false;
    float alpha[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float pv[4];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float mx = fmaxf(sc[nt][e], sc[nt][e + 2]);
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
        const float m_new = fmaxf(m_run[nt][e], mx);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        alpha[nt][e] = fast_exp2(m_run[nt][e] - m_use);
        changed |= (m_new != m_run[nt][e]);
        m_run[nt][e] = m_new;
        pv[e] = fast_exp2(sc[nt][e] - m_use);
        pv[e + 2] = fast_exp2(sc[nt][e + 2] - m_use);
        l_run[nt][e] = l_run[nt][e] * alpha[nt][e] + pv[e] + pv[e + 2];
      }
      pb[nt][0] = movmatrix_trans(pack_f16x2(pv[0], pv[1]));  // tokens 0..7
      pb[nt][1] = movmatrix_trans(pack_f16x2(pv[2], pv[3]));  // tokens 8..15
    }
    if (__any_sync(kFull, changed)) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          acc[mt][nt][0] *= alpha[nt][0];
          acc[mt][nt][1] *= alpha[nt][1];
          acc[mt][nt][2] *= alpha[nt][0];
          acc[mt][nt][3] *= alpha[nt][1];
        }
    }

    // O^T += V^T . P^T (A7); head dims of m-tile mt: VB*g8 + 2mt (+1)
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int wi = mt >> 1;
      const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
      uint32_t a0, a1, a2, a3;
      e4m3x4_to_f16x2x2(__byte_perm(x.vword(0, wi), x.vword(1, wi), sel), a0, a1);
      e4m3x4_to_f16x2x2(__byte_perm(x.vword(2, wi), x.vword(3, wi), sel), a2, a3);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_16816(acc[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
    }
  };

  // ---- main loop over this warp's units through the TMA ring
  if (lane == 0) {
    for (int i = 0; i < S && i < n_my; ++i) issue(i);
  }
  int consumed = 0;
  bool aborted = false;
#pragma unroll 1
  for (int i = 0; i < n_my; ++i) {
    const int st = i % S;
    if (!mbar_wait_bounded(&bars[warp * S + st], (uint32_t)((i / S) & 1), kWaitLimitNs)) {
      aborted = true;
      break;
    }
    consumed = i + 1;
    const int t0 = unit_t0(i);
    if (s_pid[t0 / p.ps - pg_begin] >= 0) {
      const uint8_t* kt = ring + (size_t)(warp * S + st) * STAGE;
      Frag<D> x;
      x.load(kt, kt + TILE, g8, c);
      compute_unit(t0, x);
    }
    __syncwarp();
    if (lane == 0 && i + S < n_my) {
      fence_proxy_async_smem();
      issue(i + S);
    }
  }
  if (__any_sync(kFull, aborted)) {
    if (lane == 0) atomicOr(p.err, ATLAS_DEVERR_TIMEOUT);
    // drain the loads still in flight (issued: i < min(n_my, consumed + S)), bounded
    for (int i = consumed; i < n_my && i < consumed + S; ++i)
      mbar_wait_bounded(&bars[warp * S + i % S], (uint32_t)((i / S) & 1), kWaitLimitNs);
  }
  __syncthreads();  // every warp is done with the ring: reuse it for the combine

  // ---- per-warp state to shared memory
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float l = l_run[nt][e];
      l += __shfl_xor_sync(kFull, l, 4);
      l += __shfl_xor_sync(kFull, l, 8);
      l += __shfl_xor_sync(kFull, l, 16);
      if (g8 == 0) {
        s_m[warp * RB + 8 * nt + 2 * c + e] = m_run[nt][e];
        s_l[warp * RB + 8 * nt + 2 * c + e] = l;
      }
    }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float* dst = s_o + ((size_t)warp * RB + 8 * nt + 2 * c + e) * D + VB * g8 + 2 * mt;
        *reinterpret_cast<float2*>(dst) = make_float2(acc[mt][nt][e], acc[mt][nt][e + 2]);
      }
  __syncthreads();

  // ---- combine the warps; write output (one split) or the split partial
  const float vs = __ldg(p.v_scale + h);
  const int rows_all = p.q_len * p.Hq;
  for (int idx = tid; idx < rows_here * D; idx += kThreads) {
    const int lr = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, s_m[w * RB + lr]);
    float den = 0.f, num = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = fast_exp2(s_m[w * RB + lr] - M);
        den += f * s_l[w * RB + lr];
        num += f * s_o[((size_t)w * RB + lr) * D + d];
      }
    }
    const int r = row0 + lr;
    const int i = r / p.G, hq = h * p.G + r % p.G;
    const int grow = i * p.Hq + hq;
    if (n_split_b == 1) {
      p.out[(((size_t)b * p.q_len + i) * p.Hq + hq) * D + d] =
          __float2bfloat16_rn(den > 0.f ? num / den * vs : 0.f);
    } else {
      const size_t base = ((size_t)b * p.num_splits + split) * rows_all + grow;
      p.part_o[base * D + d] = (den > 0.f) ? num / den : 0.f;
      if (d == 0) p.part_lse[base] = (den > 0.f) ? M + __log2f(den) : -INFINITY;
    }
  }
  if (n_split_b == 1) return;

  // ---- last CTA of this (b, h, rb) merges the splits (A8 -> A9)
  __threadfence();
  __syncthreads();
  int32_t* counter = p.counters + ((size_t)b * p.Hkv + h) * p.row_blocks + rb;
  if (tid == 0) s_is_last = (atomicAdd(counter, 1) == n_split_b - 1);
  __syncthreads();
  if (!s_is_last) return;
  __threadfence();

  for (int lr = warp; lr < rows_here; lr += kWarps) {
    const int r = row0 + lr;
    const int i = r / p.G, hq = h * p.G + r % p.G;
    const int grow = i * p.Hq + hq;
    const float* lse = p.part_lse + (size_t)b * p.num_splits * rows_all + grow;
    float M = -INFINITY;
    for (int sp = lane; sp < n_split_b; sp += 32) M = fmaxf(M, __ldcg(lse + (size_t)sp * rows_all));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
    float den = 0.f;
    for (int sp = lane; sp < n_split_b; sp += 32)
      den += fast_exp2(__ldcg(lse + (size_t)sp * rows_all) - M);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(kFull, den, o);
    const float inv = vs / den;
    for (int d0 = lane * 4; d0 < D; d0 += 128) {
      float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int sp = 0; sp < n_split_b; ++sp) {
        const float wgt = fast_exp2(__ldcg(lse + (size_t)sp * rows_all) - M);
        const float4 v = __ldcg(reinterpret_cast<const float4*>(
            p.part_o + (((size_t)b * p.num_splits + sp) * rows_all + grow) * D + d0));
        o4.x += wgt * v.x; o4.y += wgt * v.y; o4.z += wgt * v.z; o4.w += wgt * v.w;
      }
      __nv_bfloat16* dst = p.out + (((size_t)b * p.q_len + i) * p.Hq + hq) * D + d0;
      const __nv_bfloat162 lo = __floats2bfloat162_rn(o4.x * inv, o4.y * inv);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(o4.z * inv, o4.w * inv);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t*>(&lo);
      pk.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(dst) = pk;
    }
  }
  if (tid == 0) *counter = 0;  // ready for the next call on this stream
}

template <int D, int NT, int S>
cudaError_t launch_t(const DecodeParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                     cudaStream_t stream) {
  const size_t smem = smem_plan(D, S, p.split_tokens).total;
  auto kern = paged_decode_mma_kernel<D, NT, S>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.num_splits * p.row_blocks, p.Hkv, p.B);
  kern<<<grid, kThreads, smem, stream>>>(p, tmK, tmV);
  return cudaGetLastError();
}

template <int D, int NT>
cudaError_t launch_s(const DecodeParams& p, int stages, const CUtensorMap& tmK,
                     const CUtensorMap& tmV, cudaStream_t stream) {
  if (stages == 3) return launch_t<D, NT, 3>(p, tmK, tmV, stream);
  if (stages == 4) return launch_t<D, NT, 4>(p, tmK, tmV, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

size_t decode_mma_smem_bytes(int D, int stages, int split_tokens) {
  return smem_plan(D, stages, split_tokens).total;
}

cudaError_t launch_decode_mma(const DecodeParams& p, int rows_per_cta, int stages,
                              const CUtensorMap& tmK, const CUtensorMap& tmV,
                              cudaStream_t stream) {
  if (p.D == 128 && rows_per_cta == 8) return launch_s<128, 1>(p, stages, tmK, tmV, stream);
  if (p.D == 128 && rows_per_cta == 16) return launch_s<128, 2>(p, stages, tmK, tmV, stream);
  if (p.D == 64 && rows_per_cta == 8) return launch_s<64, 1>(p, stages, tmK, tmV, stream);
  if (p.D == 64 && rows_per_cta == 16) return launch_s<64, 2>(p, stages, tmK, tmV, stream);
  return cudaErrorInvalidValue;
}

}  // namespace atlas
