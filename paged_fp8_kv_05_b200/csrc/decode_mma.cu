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
// Per 16-token unit a warp issues, per thread, 4 + 4 coalesced 16-byte loads
// straight from the page into registers (no shared-memory staging: every
// byte is used by exactly one thread), converts E4M3 -> f16 exactly with
// cvt.rn.f16x2.e4m3x2, and runs both contractions on the tensor cores with
// mma.sync m16n8k16 (f16 in, f32 accumulate), tokens on the M side:
//   S^T[16 tok x 8 rows]  = K_tile[16 x D] . Q^T[D x 8]
//   O^T[D x 8 rows]      += V_tile^T[D x 16] . P^T[16 x 8]
// The head dimension is permuted consistently between K and Q (any
// permutation leaves q.k unchanged) so each thread's K fragment is two
// contiguous 16-byte slices of a token row; for V the thread's 16-byte slice
// of one token is interleaved with the next token's by byte_perm to form the
// token-pair registers the A operand needs.  P moves from the S^T
// accumulator layout to the PV B-operand layout with one movmatrix.trans.
#include <float.h>
#include <math.h>

#include "atlas_internal.cuh"

namespace atlas {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr unsigned kFull = 0xFFFFFFFFu;

template <int D>
struct VSlice;  // one thread's V bytes of one token: D/8 bytes
template <>
struct VSlice<128> {
  uint4 v;
  __device__ __forceinline__ uint32_t word(int i) const {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
  }
  __device__ __forceinline__ void load(const uint8_t* p) { v = ld_stream16(p); }
  __device__ __forceinline__ void zero() { v = make_uint4(0, 0, 0, 0); }
};
template <>
struct VSlice<64> {
  uint2 v;
  __device__ __forceinline__ uint32_t word(int i) const { return i == 0 ? v.x : v.y; }
  __device__ __forceinline__ void load(const uint8_t* p) { v = ld_stream8(p); }
  __device__ __forceinline__ void zero() { v = make_uint2(0, 0); }
};

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

template <int D>
struct Unit {
  static constexpr int NCH = D / 64;  // 16-byte K slices per token per thread
  uint4 k[2][NCH];                    // tokens g8 and g8 + 8
  VSlice<D> v[4];                     // tokens 2c, 2c+1, 2c+8, 2c+9
};

struct SmemLayout {
  int pid_off, m_off, l_off, o_off, total_floats;
};

__host__ __device__ inline SmemLayout smem_layout(int D, int RB, int split_tokens) {
  SmemLayout s;
  const int pid_slots = split_tokens / 16 + 2;
  s.pid_off = 0;
  s.m_off = (pid_slots + 3) & ~3;
  s.l_off = s.m_off + kWarps * RB;
  s.o_off = s.l_off + kWarps * RB;
  s.total_floats = s.o_off + kWarps * RB * D;
  return s;
}

template <int D, int NT>
__global__ void __launch_bounds__(kThreads, NT == 1 ? 3 : 2) paged_decode_mma_kernel(const DecodeParams p) {
  constexpr int RB = 8 * NT;   // query rows per CTA
  constexpr int NCH = D / 64;  // K 16-byte slices per token per thread
  constexpr int KS = D / 16;   // k-steps of QK^T
  constexpr int MT = D / 16;   // m-tiles of O^T (head dims)
  constexpr int VB = D / 8;    // V bytes per token per thread

  extern __shared__ float smem[];
  const SmemLayout lay = smem_layout(D, RB, p.split_tokens);
  int* s_pid = reinterpret_cast<int*>(smem + lay.pid_off);
  float* s_m = smem + lay.m_off;
  float* s_l = smem + lay.l_off;
  float* s_o = smem + lay.o_off;
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

  __syncthreads();

  const int n_units = (t_end - t_begin + 15) / 16;
  const size_t head_stride = (size_t)p.ps * D;

  auto load_unit = [&](int u, Unit<D>& x) {
    const int t0 = t_begin + 16 * u;
    const int pid = s_pid[t0 / p.ps - pg_begin];
    if (pid < 0) return;  // skipped at compute time
    const size_t off = ((size_t)pid * p.Hkv + h) * head_stride + (size_t)(t0 % p.ps) * D;
    const uint8_t* kb = p.k_pages + off;
    const uint8_t* vb = p.v_pages + off;
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
      x.k[0][j] = ld_stream16(kb + g8 * D + j * 64 + 16 * c);
      x.k[1][j] = ld_stream16(kb + (g8 + 8) * D + j * 64 + 16 * c);
    }
    x.v[0].load(vb + (2 * c) * D + VB * g8);
    x.v[1].load(vb + (2 * c + 1) * D + VB * g8);
    x.v[2].load(vb + (2 * c + 8) * D + VB * g8);
    x.v[3].load(vb + (2 * c + 9) * D + VB * g8);
  };

  auto compute_unit = [&](int u, Unit<D>& x) {
    const int t0 = t_begin + 16 * u;
    if (s_pid[t0 / p.ps - pg_begin] < 0) return;  // bad page id: tokens skipped

    // S^T = K . Q^T  (A3 dequant-to-f16 + A4)
    float sacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t a0, a1, a2, a3;
      e4m3x4_to_f16x2x2(word_of(x.k[0][ks / 4], ks % 4), a0, a2);
      e4m3x4_to_f16x2x2(word_of(x.k[1][ks / 4], ks % 4), a1, a3);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_16816(sacc[nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
    }

    // scale into the log2 domain, causal / tail mask (A5)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] *= scale2;
    if (t0 + 15 > min_lim) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tok = t0 + g8 + ((e & 2) ? 8 : 0);
          if (tok > lim[nt][e & 1]) sacc[nt][e] = -INFINITY;
        }
    }
    if (t0 + 16 > L) {  // tail of the last page: no V garbage may reach P*V
      if (t0 + 2 * c >= L) x.v[0].zero();
      if (t0 + 2 * c + 1 >= L) x.v[1].zero();
      if (t0 + 2 * c + 8 >= L) x.v[2].zero();
      if (t0 + 2 * c + 9 >= L) x.v[3].zero();
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
        float mx = fmaxf(sacc[nt][e], sacc[nt][e + 2]);
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
        const float m_new = fmaxf(m_run[nt][e], mx);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        alpha[nt][e] = fast_exp2(m_run[nt][e] - m_use);
        changed |= (m_new != m_run[nt][e]);
        m_run[nt][e] = m_new;
        pv[e] = fast_exp2(sacc[nt][e] - m_use);
        pv[e + 2] = fast_exp2(sacc[nt][e + 2] - m_use);
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
      e4m3x4_to_f16x2x2(__byte_perm(x.v[0].word(wi), x.v[1].word(wi), sel), a0, a1);
      e4m3x4_to_f16x2x2(__byte_perm(x.v[2].word(wi), x.v[3].word(wi), sel), a2, a3);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_16816(acc[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
    }
  };

  // ---- main loop: register double buffer, one unit in flight ahead
  {
    Unit<D> cur, nxt;
    int u = warp;
    if (u < n_units) load_unit(u, cur);
#pragma unroll 1
    for (; u < n_units; u += kWarps) {
      if (u + kWarps < n_units) load_unit(u + kWarps, nxt);
      compute_unit(u, cur);
      cur = nxt;
    }
  }

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

template <int D, int NT>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t stream) {
  const SmemLayout lay = smem_layout(D, 8 * NT, p.split_tokens);
  const size_t smem = (size_t)lay.total_floats * sizeof(float);
  auto kern = paged_decode_mma_kernel<D, NT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.num_splits * p.row_blocks, p.Hkv, p.B);
  kern<<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t decode_mma_smem_bytes(int D, int rows_per_cta, int split_tokens) {
  return (size_t)smem_layout(D, rows_per_cta, split_tokens).total_floats * sizeof(float);
}

cudaError_t launch_decode_mma(const DecodeParams& p, int rows_per_cta, cudaStream_t stream) {
  if (p.D == 128 && rows_per_cta == 8) return launch_t<128, 1>(p, stream);
  if (p.D == 128 && rows_per_cta == 16) return launch_t<128, 2>(p, stream);
  if (p.D == 64 && rows_per_cta == 8) return launch_t<64, 1>(p, stream);
  if (p.D == 64 && rows_per_cta == 16) return launch_t<64, 2>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace atlas
