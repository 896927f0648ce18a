// Paged FP8 decode / MTP-verify grouped-query attention on the FP8 tensor cores.
//
// Computes, for every sequence b, KV head h and query row r = (i, g) of the
// head's group (i < q_len new tokens, g < G = Hq/Hkv q-heads per KV head):
//     s_t = sm_scale * k_scale[h] * sum_d q[b,i,h*G+g,d] * code(K[t,h,d])
//     out = v_scale[h] * sum_t softmax(s)_t * code(V[t,h,:]),   t <= L_b - q_len + i
// i.e. the plain masked SDPA over the dequantised cache with the two per-head
// scales factored out of the dot products.  Sources: the FlashAttention-2-style
// online softmax and the dedicated MQA/GQA kernels of the Atlas deep-dive
// (ainews.cool, "Attention" paragraph), its FP8 with scale factors
// ("Quantisation" paragraph), the fixed-size KV blocks ("Memory architecture"
// paragraph) and the paged FP8 KV cache with MTP K = 4 verify of the GB10 page
// (ainews.surl.tw).
//
// Arithmetic.  Both contractions run on mma.sync m16n8k32 with E4M3 operands
// and f32 accumulation, tokens on the M side; the cached codes are consumed
// as they are (no conversion):
//   S^T[16 tok x 8 rows]  = K_tile[16 x 32] . (Qhi + Qlo)^T[32 x 8]   per 32 dims
//   O^T[16 dims x 8 rows] += V_tile^T[16 x 32] . (Phi + Plo)^T[32 x 8] per 32 tokens
// The bf16 query row is scaled by a power of two a_r (max |q| a_r in (224, 448])
// and written as the sum of two E4M3 values: hi = E4M3(q a_r), lo = E4M3(q a_r - hi).
// A bf16 significand has 8 bits, hi keeps 4 and lo the next 4, so the pair is
// exact unless lo falls below the E4M3 normal range (a contribution under
// 2^-9 of the row's largest element).  The probabilities are taken as
// p = 2^(s - m + 8) in f32 (so 2^-6 <= p <= 2^8 covers the useful range),
// rounded to f16 and split the same way (hi + lo carries 8 significant bits).
// The row sum l accumulates the f32 p, and out = O / l, so the 2^8 and a_r
// factors cancel exactly.  Error budget: the 8-bit P adds ~1e-4 relative L2 to
// the bf16 output rounding (~1.7e-3) on the benchmark workloads.
//
// Fragment layouts.  The head dimension is permuted consistently between K and
// Q: k-step s = 2j + hs of 32 dims reads bytes 64j + 16c + 8hs + {0..7} of a
// token row (c = lane % 4), so each lane's K operand is two 16-byte chunks of a
// token row.  V pages are kept in 16-slot groups, head-dim-major inside a group
// ([D][16] bytes, slots interleaved so that bytes 4c..4c+3 hold slots 2c, 2c+1,
// 2c+8, 2c+9), so a V^T fragment is 4 adjacent bytes and one ldmatrix.x4
// fetches the A operand of a 16-dim m-tile for 32 tokens.  P leaves the S^T
// accumulator through movmatrix.trans, which hands each lane exactly those
// four tokens of its row -- no shuffles.
//
// Work split and staging.  CTA (split s, KV head h, sequence b, row group)
// owns the KV tokens [s*T, min((s+1)*T, L_b)) and RBG blocks of 8*NT query rows.
// Its 4 warps form 4/RBG streams; the RBG warps of a stream share one ring of S
// shared-memory stages, each holding the K tiles and V^T tiles of one 32-token
// unit (two 16-token page pieces, each a contiguous block of 16*D bytes in its
// page), filled by 1-D bulk copies (cp.async.bulk, no multicast) completing
// on a "full" mbarrier; with RBG > 1 an "empty" mbarrier counts the
// consumers before a stage is refilled.  Streams take units round-robin with
// private online-softmax state and are combined in shared memory.  A sequence
// with one split writes bf16 output directly; otherwise each split writes
// (O/l, log2-sum-exp) to the workspace and the CTA that finishes a
// (b, h, row group) last -- one atomic counter, no waiting -- merges the splits
// and resets the counter.  Every mbarrier wait is bounded (200 ms of wall
// clock): a wait that runs out flags ATLAS_DEVERR_TIMEOUT and the warp stops
// computing after draining the loads it issued.
#include <float.h>
#include <math.h>

#include "atlas_internal.cuh"

namespace atlas {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr uint64_t kWaitLimitNs = 200ull * 1000 * 1000;
constexpr int kUnit = 32;  // tokens per pipeline unit (two 16-token tiles)

// ---------------------------------------------------------------- PTX wrappers

// D += A * B, m16n8k32, E4M3 inputs, f32 accumulate.
__device__ __forceinline__ void mma_e4m3(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two f32 -> two E4M3 (round to nearest even, saturating); `lo` in the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// f16x2 -> E4M3x2 (low half -> low byte), round to nearest even, saturating.
__device__ __forceinline__ uint32_t f16x2_to_e4m3x2(uint32_t x) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(r) : "r"(x));
  return r;
}

// E4M3x2 (low byte first) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t x16) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
      : "=r"(r)
      : "r"(x16));
  return r;
}

__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                            uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Split two f16x2 words (4 values, in k order) into E4M3x4 hi and lo words:
// hi = E4M3(x), lo = E4M3(x - hi).  The subtraction is exact in f16.
__device__ __forceinline__ void split_e4m3x4(uint32_t w0, uint32_t w1, uint32_t& hi,
                                             uint32_t& lo) {
  const uint32_t h0 = f16x2_to_e4m3x2(w0), h1 = f16x2_to_e4m3x2(w1);
  const uint32_t l0 = f16x2_to_e4m3x2(hsub2(w0, e4m3x2_to_f16x2(h0)));
  const uint32_t l1 = f16x2_to_e4m3x2(hsub2(w1, e4m3x2_to_f16x2(h1)));
  hi = h0 | (h1 << 16);
  lo = l0 | (l1 << 16);
}

// Byte mask of a V^T fragment word (bytes 4c..4c+3 of a 16-slot group row,
// holding slots 2c, 2c+1, 2c+8, 2c+9) keeping the slots below `nvalid`.
__device__ __forceinline__ uint32_t token_mask4(int nvalid, int c) {
  return (2 * c < nvalid ? 0x000000FFu : 0u) | (2 * c + 1 < nvalid ? 0x0000FF00u : 0u) |
         (2 * c + 8 < nvalid ? 0x00FF0000u : 0u) | (2 * c + 9 < nvalid ? 0xFF000000u : 0u);
}

// ----------------------------------------------------------- shared memory plan

template <int D, int S, int NSTREAM, int RC>
struct Smem {
  static constexpr int TILE = 16 * D;     // one 16-token K tile or V^T tile
  static constexpr int STAGE = 4 * TILE;  // K_A, K_B, V_A, V_B
  static constexpr size_t RING = (size_t)NSTREAM * S * STAGE;
  // stream-combine buffers (m, l, O) reuse the ring after the main loop
  static constexpr size_t COMBINE = NSTREAM > 1 ? (size_t)NSTREAM * RC * (D + 2) * 4 : 0;
  static constexpr size_t REGION = RING > COMBINE ? RING : (COMBINE + 1023) / 1024 * 1024;
  static constexpr size_t BARS = REGION;                            // full[], empty[]
  static constexpr size_t PIDS = BARS + (size_t)2 * NSTREAM * S * 8;
  static size_t total(int split_tokens) { return PIDS + (size_t)(split_tokens / 16 + 2) * 4 + 1024; }
};

// ------------------------------------------------------------------- the kernel

template <int D, int NT, int RBG, int S>
__global__ void __launch_bounds__(kThreads, NT == 1 ? 3 : 2)
    paged_decode_fp8_kernel(const DecodeParams p) {
  constexpr int RW = 8 * NT;             // query rows per warp
  constexpr int RC = RW * RBG;           // query rows per CTA
  constexpr int NSTREAM = kWarps / RBG;  // unit streams per CTA
  constexpr int NCH = D / 64;            // 16-byte K chunks per token per lane
  constexpr int KSTEP = D / 32;          // k-steps of QK^T
  constexpr int MT = D / 16;             // m-tiles of O^T
  using SM = Smem<D, S, NSTREAM, RC>;
  constexpr int TILE = SM::TILE;
  constexpr int STAGE = SM::STAGE;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + SM::BARS);
  uint64_t* empty_bar = full_bar + NSTREAM * S;
  int* s_piece = reinterpret_cast<int*>(smem + SM::PIDS);
  __shared__ int s_is_last;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, c = lane & 3;
  const int stream = warp / RBG, rbw = warp % RBG;
  const int n_groups = p.row_blocks;  // row groups of RC rows per (b, h)
  const int grp = blockIdx.x % n_groups;
  const int split = blockIdx.x / n_groups;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int L = __ldg(p.seq_lens + b);
  const int Rtot = p.q_len * p.G;
  const int cta_row0 = grp * RC;
  const int rows_cta = min(RC, Rtot - cta_row0);
  const int row0 = cta_row0 + rbw * RW;  // this warp's first row

  // ---- invalid sequence: zero this CTA's rows once (split 0) and flag it
  if (L < p.q_len || L > p.max_blocks * p.ps || L > p.num_splits * p.split_tokens) {
    if (split == 0) {
      if (tid == 0) atomicOr(p.err, ATLAS_DEVERR_SEQ_LEN);
      for (int idx = tid; idx < rows_cta * D; idx += kThreads) {
        const int r = cta_row0 + idx / D, d = idx % D;
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

  // ---- A0, fused append: quantise and store the step's new tokens that fall in
  // this split (positions L - q_len .. L - 1), then order those global writes
  // before the bulk copies that read the pages back
  if (p.k_new != nullptr) {
    const int first_new = L - p.q_len;
    const int a0 = max(t_begin, first_new);
    const int n_tok = t_end - a0;
    if (n_tok > 0) {
      constexpr int CH = D / 16;
      for (int idx = tid; idx < 2 * n_tok * CH; idx += kThreads) {
        const int which = idx / (n_tok * CH);  // 0 = K, 1 = V
        const int r = idx - which * n_tok * CH;
        const int pos = a0 + r / CH, j = r % CH;
        const int page = __ldg(p.block_table + (size_t)b * p.max_blocks + pos / p.ps);
        if (page < 0 || page >= p.num_pages) {
          atomicOr(p.err, ATLAS_DEVERR_APPEND);
          continue;
        }
        float x[16];
        load16_as_f32(which ? p.v_new : p.k_new,
                      (((size_t)b * p.q_len + (pos - first_new)) * p.Hkv + h) * D + 16 * j,
                      p.new_dtype, x);
        const uint4 codes = quantize16_e4m3(x, __ldg((which ? p.v_scale : p.k_scale) + h));
        const size_t head_page = (size_t)page * p.Hkv + h;
        if (!which)
          store16_k(const_cast<uint8_t*>(p.k_pages), head_page, D, p.ps, pos % p.ps, j, codes);
        else
          store16_v(const_cast<uint8_t*>(p.v_pages), head_page, D, p.ps, pos % p.ps, j, codes);
      }
      __threadfence();
      fence_proxy_async_global();
    }
  }

  // ---- A2, block-table gather: index of every 16-token piece of this split,
  // counted in 16*D-byte blocks of the page arrays (-1 for a bad page id).
  // Piece k holds tokens [t_begin + 16k, +16): page (t / ps), slot group
  // (t % ps) / 16; the divisions happen here once, not per unit.
  const int n_pieces = (t_end - t_begin + 15) / 16;
  const int groups_per_page = p.ps / 16;
  for (int k = tid; k < n_pieces; k += kThreads) {
    const int t = t_begin + 16 * k;
    const int pg = t / p.ps;
    int pid = __ldg(p.block_table + (size_t)b * p.max_blocks + pg);
    int piece = -1;
    if (pid < 0 || pid >= p.num_pages) {
      atomicOr(p.err, ATLAS_DEVERR_PAGE_ID);
    } else {
      piece = (pid * p.Hkv + h) * groups_per_page + (t - pg * p.ps) / 16;
    }
    s_piece[k] = piece;
  }
  if (tid < NSTREAM * S) {
    mbar_init(&full_bar[tid], 1);
    mbar_init(&empty_bar[tid], RBG);
  }
  if (tid == 0) fence_mbar_init();

  __syncthreads();  // page ids and barrier init visible

  // this stream's units: u = stream + NSTREAM * i, i < n_my
  const int n_units = (t_end - t_begin + kUnit - 1) / kUnit;
  const int n_my = (stream < n_units) ? (n_units - stream + NSTREAM - 1) / NSTREAM : 0;
  const bool producer = (rbw == 0) && (lane == 0);
  auto unit_t0 = [&](int i) { return t_begin + kUnit * (stream + NSTREAM * i); };
  // pieces of unit i: 2(stream + NSTREAM i) and the next one (if inside the split)
  auto piece_of = [&](int k) { return k < n_pieces ? s_piece[k] : -1; };

  constexpr size_t kPiece = (size_t)16 * D;  // bytes of one 16-token piece
  auto issue = [&](int i) {  // producer lane only: stage i % S <- unit i
    const int st = i % S;
    const int k = 2 * (stream + NSTREAM * i);
    uint64_t* bar = &full_bar[stream * S + st];
    uint8_t* dst = ring + (size_t)(stream * S + st) * STAGE;
    const int pa = piece_of(k), pb = piece_of(k + 1);
    const uint32_t bytes = (pa >= 0 ? 2 * TILE : 0) + (pb >= 0 ? 2 * TILE : 0);
    if (bytes == 0) {
      mbar_arrive(bar);
      return;
    }
    mbar_arrive_expect_tx(bar, bytes);
    // a 16-token piece is TILE contiguous bytes in both layouts: K rows
    // (slot0 .. slot0 + 15) x D, and V group slot0 / 16 ([D][16])
    if (pa >= 0) {
      bulk_load(dst, p.k_pages + (size_t)pa * kPiece, TILE, bar);
      bulk_load(dst + 2 * TILE, p.v_pages + (size_t)pa * kPiece, TILE, bar);
    }
    if (pb >= 0) {
      bulk_load(dst + TILE, p.k_pages + (size_t)pb * kPiece, TILE, bar);
      bulk_load(dst + 3 * TILE, p.v_pages + (size_t)pb * kPiece, TILE, bar);
    }
  };


  // the first S units of every stream go out before the query is prepared,
  // so their loads overlap the Q fetch and split below
  if (producer) {
    for (int i = 0; i < S && i < n_my; ++i) issue(i);
  }

  // ---- Q^T fragments as E4M3 hi + lo with a per-row power-of-two scale
  // B operand of k-step s = 2j + hs: b0 = dims 64j+16c+8hs+{0..3}, b1 = +{4..7}.
  uint32_t qhi[NT][KSTEP][2], qlo[NT][KSTEP][2];
  float alpha_row[NT];  // the scale of row 8nt + g8
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int r = row0 + 8 * nt + g8;
    float x[NCH][16];
    if (r < Rtot) {
      const int i = r / p.G, hq = h * p.G + r % p.G;
      const __nv_bfloat16* qrow = p.q + (((size_t)b * p.q_len + i) * p.Hq + hq) * D;
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        const uint4* src = reinterpret_cast<const uint4*>(qrow + j * 64 + 16 * c);
        const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
        const uint32_t wv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          x[j][2 * k] = __uint_as_float(wv[k] << 16);
          x[j][2 * k + 1] = __uint_as_float(wv[k] & 0xFFFF0000u);
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < NCH; ++j)
#pragma unroll
        for (int k = 0; k < 16; ++k) x[j][k] = 0.f;
    }
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < NCH; ++j)
#pragma unroll
      for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(x[j][k]));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
    // a = 2^(135 - e) puts amax in [256, 512); halve it if amax * a > 448
    const int e = (int)((__float_as_uint(amax) >> 23) & 0xFF);
    float a = 1.f;
    if (amax > 0.f) {
      const int ex = min(254, max(1, 262 - e));
      a = __uint_as_float((uint32_t)ex << 23);
      if (amax * a > 448.f) a *= 0.5f;
    }
    alpha_row[nt] = a;
#pragma unroll
    for (int j = 0; j < NCH; ++j)
#pragma unroll
      for (int hs = 0; hs < 2; ++hs)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int k0 = 8 * hs + 4 * half;
          const float y0 = x[j][k0] * a, y1 = x[j][k0 + 1] * a;
          const float y2 = x[j][k0 + 2] * a, y3 = x[j][k0 + 3] * a;
          const uint32_t h01 = f32x2_to_e4m3x2(y0, y1), h23 = f32x2_to_e4m3x2(y2, y3);
          const uint32_t f01 = e4m3x2_to_f16x2(h01), f23 = e4m3x2_to_f16x2(h23);
          const float2 b01 = __half22float2(*reinterpret_cast<const __half2*>(&f01));
          const float2 b23 = __half22float2(*reinterpret_cast<const __half2*>(&f23));
          const uint32_t l01 = f32x2_to_e4m3x2(y0 - b01.x, y1 - b01.y);
          const uint32_t l23 = f32x2_to_e4m3x2(y2 - b23.x, y3 - b23.y);
          qhi[nt][2 * j + hs][half] = h01 | (h23 << 16);
          qlo[nt][2 * j + hs][half] = l01 | (l23 << 16);
        }
  }

  // ---- per accumulator row (8nt + 2c + e): causal limit and score scale
  const float kscale = __ldg(p.k_scale + h) * p.qk_scale_log2;
  int lim[NT][2];
  float scale2[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int r = row0 + 8 * nt + 2 * c + e;
      lim[nt][e] = (r < Rtot) ? (L - p.q_len + r / p.G) : (L - 1);
      const float a = __shfl_sync(kFull, alpha_row[nt], 4 * (2 * c + e));
      scale2[nt][e] = kscale / a;
    }
  const int min_lim = L - p.q_len + row0 / p.G;

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

  // this lane's K operand words of one 16-token K tile: rows g8 and g8 + 8,
  // 16-byte chunks 4j + c (D = 128: odd rows fetch their chunks in the other
  // order, which keeps the 8 lanes of each shared-memory phase on distinct banks)
  auto load_k = [&](const uint8_t* kt, uint4 (&kr)[2][NCH]) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int row = g8 + 8 * t;
      if constexpr (D == 128) {
        const int ja = g8 & 1;
        const uint8_t* rb = kt + row * 128;
        const uint4 x0 = *reinterpret_cast<const uint4*>(rb + ((4 * ja + c) << 4));
        const uint4 x1 = *reinterpret_cast<const uint4*>(rb + ((4 * (1 - ja) + c) << 4));
        kr[t][0] = ja ? x1 : x0;
        kr[t][1] = ja ? x0 : x1;
      } else {
        kr[t][0] = *reinterpret_cast<const uint4*>(kt + row * 64 + (c << 4));
      }
    }
  };

  // S^T for the two 16-token K tiles of a unit: hi and lo parts of Q in separate
  // accumulators, so four independent mma chains interleave
  auto qk_unit = [&](const uint8_t* stage, float (&sa)[NT][4], float (&sb)[NT][4]) {
    uint4 ka[2][NCH], kb[2][NCH];
    load_k(stage, ka);
    load_k(stage + TILE, kb);
    float ah[NT][4], al[NT][4], bh[NT][4], bl[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) ah[nt][e] = al[nt][e] = bh[nt][e] = bl[nt][e] = 0.f;
#pragma unroll
    for (int j = 0; j < NCH; ++j)
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        const int ks = 2 * j + hs;
        const uint32_t a0 = hs ? ka[0][j].z : ka[0][j].x, a2 = hs ? ka[0][j].w : ka[0][j].y;
        const uint32_t a1 = hs ? ka[1][j].z : ka[1][j].x, a3 = hs ? ka[1][j].w : ka[1][j].y;
        const uint32_t c0 = hs ? kb[0][j].z : kb[0][j].x, c2 = hs ? kb[0][j].w : kb[0][j].y;
        const uint32_t c1 = hs ? kb[1][j].z : kb[1][j].x, c3 = hs ? kb[1][j].w : kb[1][j].y;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_e4m3(ah[nt], a0, a1, a2, a3, qhi[nt][ks][0], qhi[nt][ks][1]);
          mma_e4m3(bh[nt], c0, c1, c2, c3, qhi[nt][ks][0], qhi[nt][ks][1]);
          mma_e4m3(al[nt], a0, a1, a2, a3, qlo[nt][ks][0], qlo[nt][ks][1]);
          mma_e4m3(bl[nt], c0, c1, c2, c3, qlo[nt][ks][0], qlo[nt][ks][1]);
        }
      }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        sa[nt][e] = ah[nt][e] + al[nt][e];
        sb[nt][e] = bh[nt][e] + bl[nt][e];
      }
  };

  auto compute_unit = [&](int i, const uint8_t* stage) {
    const int t0 = unit_t0(i);
    const int k = 2 * (stream + NSTREAM * i);
    const int nvA = (piece_of(k) >= 0) ? min(16, t_end - t0) : 0;
    const int nvB = (piece_of(k + 1) >= 0) ? min(16, t_end - t0 - 16) : 0;
    float sa[NT][4], sb[NT][4];
    qk_unit(stage, sa, sb);

    // causal / tail / skipped-page mask (A5)
    const bool tail = (nvA < 16) || (nvB < 16);
    if (tail || t0 + kUnit - 1 > min_lim) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int tl = g8 + ((e & 2) ? 8 : 0);
          if (tl >= nvA || t0 + tl > lim[nt][e & 1]) sa[nt][e] = -INFINITY;
          if (tl >= nvB || t0 + 16 + tl > lim[nt][e & 1]) sb[nt][e] = -INFINITY;
        }
    }

    // online softmax (A6) over the 32 tokens, p = 2^(s - m + 8) with m the running
    // reference of the row.  A row's reference only moves (to the exact row max,
    // rescaling its O and l) when one of its scores exceeds it by more than 0.5,
    // so p <= 2^8.5 < 448 and the common step needs no cross-lane max.
    bool need = false;
    float lmax[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        lmax[nt][e] = fmaxf(fmaxf(sa[nt][e], sa[nt][e + 2]), fmaxf(sb[nt][e], sb[nt][e + 2])) *
                      scale2[nt][e];
        need |= lmax[nt][e] > m_run[nt][e] + 0.5f;
      }
    if (__any_sync(kFull, need)) {
      float alpha[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float mx = lmax[nt][e];
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
          // decided per row (mx is uniform over the row's lanes), so a row's
          // reference -- and its bits -- never depend on the other rows
          const bool move = mx > m_run[nt][e] + 0.5f;
          const float m_new = move ? mx : m_run[nt][e];
          alpha[nt][e] = move ? fast_exp2(m_run[nt][e] - m_new) : 1.f;
          m_run[nt][e] = m_new;
          l_run[nt][e] *= alpha[nt][e];
        }
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
    // P^T B operand for row g8: movmatrix leaves tokens (2c, 2c+1) and (8+2c, 9+2c)
    // of a 16-token tile in this lane -- exactly the slots of V^T bytes 4c..4c+3
    uint32_t pbhi[NT][2], pblo[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float pa[4], pb[4];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float sc = scale2[nt][e];
        const float off = 8.f - ((m_run[nt][e] == -INFINITY) ? 0.f : m_run[nt][e]);
        pa[e] = fast_exp2(fmaf(sa[nt][e], sc, off));
        pa[e + 2] = fast_exp2(fmaf(sa[nt][e + 2], sc, off));
        pb[e] = fast_exp2(fmaf(sb[nt][e], sc, off));
        pb[e + 2] = fast_exp2(fmaf(sb[nt][e + 2], sc, off));
        l_run[nt][e] += (pa[e] + pa[e + 2]) + (pb[e] + pb[e + 2]);
      }
      const uint32_t xa = movmatrix_trans(pack_f16x2(pa[0], pa[1]));  // toks 2c, 2c+1
      const uint32_t ya = movmatrix_trans(pack_f16x2(pa[2], pa[3]));  // toks 8+2c, 9+2c
      const uint32_t xb = movmatrix_trans(pack_f16x2(pb[0], pb[1]));
      const uint32_t yb = movmatrix_trans(pack_f16x2(pb[2], pb[3]));
      split_e4m3x4(xa, ya, pbhi[nt][0], pblo[nt][0]);
      split_e4m3x4(xb, yb, pbhi[nt][1], pblo[nt][1]);
    }

    // O^T += V^T . P^T (A7): m-tile mt = head dims 16mt + {g8, g8 + 8}
    const int mat = lane >> 3, mrow = lane & 7;
    const uint32_t vbase = smem_u32(stage + 2 * TILE + ((mat >> 1) ? TILE : 0)) +
                           (uint32_t)((8 * (mat & 1) + mrow) * 16);
    uint32_t mA = 0xFFFFFFFFu, mB = 0xFFFFFFFFu;
    if (tail) {  // slots past the end of the sequence (or of a skipped page)
      mA = token_mask4(nvA, c);
      mB = token_mask4(nvB, c);
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(vbase + mt * 256, a0, a1, a2, a3);
      if (tail) {
        a0 &= mA; a1 &= mA; a2 &= mB; a3 &= mB;
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mma_e4m3(acc[mt][nt], a0, a1, a2, a3, pbhi[nt][0], pbhi[nt][1]);
        mma_e4m3(acc[mt][nt], a0, a1, a2, a3, pblo[nt][0], pblo[nt][1]);
      }
    }
  };

  // ---- main loop over this stream's units through the staging ring
  int consumed = 0;
  bool aborted = false;
#pragma unroll 1
  for (int i = 0; i < n_my; ++i) {
    const int st = i % S;
    const uint32_t par = (uint32_t)((i / S) & 1);
    if (!mbar_wait_bounded(&full_bar[stream * S + st], par, kWaitLimitNs)) {
      aborted = true;
      break;
    }
    consumed = i + 1;
    if (row0 < Rtot) compute_unit(i, ring + (size_t)(stream * S + st) * STAGE);
    __syncwarp();
    if constexpr (RBG > 1) {
      if (lane == 0) mbar_arrive(&empty_bar[stream * S + st]);
    }
    if (producer && i + S < n_my) {
      if constexpr (RBG > 1) {
        if (!mbar_wait_bounded(&empty_bar[stream * S + st], par, kWaitLimitNs)) {
          aborted = true;
        }
      }
      if (!aborted) {
        fence_proxy_async_smem();
        issue(i + S);
      }
    }
    if (__any_sync(kFull, aborted)) break;
  }
  if (__any_sync(kFull, aborted)) {
    if (lane == 0) atomicOr(p.err, ATLAS_DEVERR_TIMEOUT);
    for (int i = consumed; i < n_my && i < consumed + S; ++i)
      mbar_wait_bounded(&full_bar[stream * S + i % S], (uint32_t)((i / S) & 1), kWaitLimitNs);
  }

  // ---- row sums over the token lanes
  float l_full[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float l = l_run[nt][e];
      l += __shfl_xor_sync(kFull, l, 4);
      l += __shfl_xor_sync(kFull, l, 8);
      l += __shfl_xor_sync(kFull, l, 16);
      l_full[nt][e] = l;
    }
  const float vs = __ldg(p.v_scale + h);
  const int rows_all = p.q_len * p.Hq;

  if constexpr (NSTREAM == 1) {
    // one stream: every warp owns its rows outright; store from registers
    if (row0 < Rtot) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int r = row0 + 8 * nt + 2 * c + e;
          if (r >= Rtot) continue;
          const int i = r / p.G, hq = h * p.G + r % p.G;
          const int grow = i * p.Hq + hq;
          const float den = l_full[nt][e];
          const float inv = den > 0.f ? 1.f / den : 0.f;
          if (n_split_b == 1) {
            __nv_bfloat16* orow = p.out + (((size_t)b * p.q_len + i) * p.Hq + hq) * D;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              orow[16 * mt + g8] = __float2bfloat16_rn(acc[mt][nt][e] * inv * vs);
              orow[16 * mt + g8 + 8] = __float2bfloat16_rn(acc[mt][nt][e + 2] * inv * vs);
            }
          } else {
            const size_t base = ((size_t)b * p.num_splits + split) * rows_all + grow;
            float* prow = p.part_o + base * D;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              prow[16 * mt + g8] = acc[mt][nt][e] * inv;
              prow[16 * mt + g8 + 8] = acc[mt][nt][e + 2] * inv;
            }
            if (g8 == 0) p.part_lse[base] = den > 0.f ? m_run[nt][e] + __log2f(den) : -INFINITY;
          }
        }
    }
  } else {
    __syncthreads();  // every warp is done with the ring: reuse it for the combine
    float* s_m = reinterpret_cast<float*>(ring);
    float* s_l = s_m + NSTREAM * RC;
    float* s_o = s_l + NSTREAM * RC;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int lr = rbw * RW + 8 * nt + 2 * c + e;
        if (g8 == 0) {
          s_m[stream * RC + lr] = m_run[nt][e];
          s_l[stream * RC + lr] = l_full[nt][e];
        }
      }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int lr = rbw * RW + 8 * nt + 2 * c + (e & 1);
          const int d = 16 * mt + g8 + ((e & 2) ? 8 : 0);
          s_o[((size_t)stream * RC + lr) * D + d] = acc[mt][nt][e];
        }
    __syncthreads();

    // combine the streams; write output (one split) or the split partial
    for (int idx = tid; idx < rows_cta * D; idx += kThreads) {
      const int lr = idx / D, d = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NSTREAM; ++w) M = fmaxf(M, s_m[w * RC + lr]);
      float den = 0.f, num = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < NSTREAM; ++w) {
          const float f = fast_exp2(s_m[w * RC + lr] - M);
          den += f * s_l[w * RC + lr];
          num += f * s_o[((size_t)w * RC + lr) * D + d];
        }
      }
      const int r = cta_row0 + lr;
      const int i = r / p.G, hq = h * p.G + r % p.G;
      const int grow = i * p.Hq + hq;
      if (n_split_b == 1) {
        p.out[(((size_t)b * p.q_len + i) * p.Hq + hq) * D + d] =
            __float2bfloat16_rn(den > 0.f ? num / den * vs : 0.f);
      } else {
        const size_t base = ((size_t)b * p.num_splits + split) * rows_all + grow;
        p.part_o[base * D + d] = (den > 0.f) ? num / den : 0.f;
        // the log2-sum-exp carries the 2^8 factor of p; it cancels in the merge
        if (d == 0) p.part_lse[base] = (den > 0.f) ? M + __log2f(den) : -INFINITY;
      }
    }
  }
  if (n_split_b == 1) return;

  // ---- last CTA of this (b, h, row group) merges the splits (A8 -> A9)
  __threadfence();
  __syncthreads();
  int32_t* counter = p.counters + ((size_t)b * p.Hkv + h) * p.row_blocks + grp;
  if (tid == 0) s_is_last = (atomicAdd(counter, 1) == n_split_b - 1);
  __syncthreads();
  if (!s_is_last) return;
  __threadfence();

  for (int lr = warp; lr < rows_cta; lr += kWarps) {
    const int r = cta_row0 + lr;
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

template <int D, int NT, int RBG, int S>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t stream) {
  const size_t smem = Smem<D, S, kWarps / RBG, 8 * NT * RBG>::total(p.split_tokens);
  auto kern = paged_decode_fp8_kernel<D, NT, RBG, S>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.num_splits * p.row_blocks, p.Hkv, p.B);
  kern<<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int D, int NT, int RBG>
cudaError_t launch_s(const DecodeParams& p, int stages, cudaStream_t stream) {
  if (stages == 2) return launch_t<D, NT, RBG, 2>(p, stream);
  if (stages == 3) return launch_t<D, NT, RBG, 3>(p, stream);
  return cudaErrorInvalidValue;
}

template <int D>
cudaError_t launch_d(const DecodeParams& p, int rows_per_warp, int rbg, int stages,
                     cudaStream_t stream) {
  if (rows_per_warp == 8 && rbg == 1) return launch_s<D, 1, 1>(p, stages, stream);
  if (rows_per_warp == 16 && rbg == 1) return launch_s<D, 2, 1>(p, stages, stream);
  if (rows_per_warp == 16 && rbg == 2) return launch_s<D, 2, 2>(p, stages, stream);
  if (rows_per_warp == 16 && rbg == 4) return launch_s<D, 2, 4>(p, stages, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_fp8(const DecodeParams& p, int rows_per_warp, int rbg, int stages,
                              cudaStream_t stream) {
  if (p.D == 128) return launch_d<128>(p, rows_per_warp, rbg, stages, stream);
  if (p.D == 64) return launch_d<64>(p, rows_per_warp, rbg, stages, stream);
  return cudaErrorInvalidValue;
}

}  // namespace atlas
