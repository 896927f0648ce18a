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
// p = 2^(s - m + 8) in f32, rounded to f16 and split the same way (hi + lo
// carries 8 significant bits).  The row sum l accumulates the f32 p, and
// out = O / l, so the 2^8 and a_r factors cancel exactly.  The 8-bit P adds
// ~1e-4 relative L2 to the bf16 output rounding (~1.7e-3) on the benchmark
// workloads.
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
// Work partition.  A segment is (sequence b, KV head h, row group rg):
// ceil(L_b / 32) units of 32 KV tokens for up to RC query rows.  Two modes
// share all code below the prologue:
//  * grid: CTA = one split of split_tokens tokens of one segment; the hardware
//    hands CTAs to SMs as slots free up;
//  * balanced: all units of all segments form one list (segments in (b, h, rg)
//    order) and CTA c of the G CTAs takes units [c*U/G, (c+1)*U/G), so every
//    CTA streams the same amount of KV whatever the length mix; its range cuts
//    the list into portions, one per segment it touches.
// The "block size adapted to sequence length and architecture" of the Atlas
// deep-dive is the host's choice of split length / range count.  The CTA's 4
// warps form 4/RBG streams that take its units round-robin; the RBG warps of a
// stream share one ring of S shared-memory stages, each holding the K and V^T
// pieces of one unit (two 16-token page pieces, each a contiguous block of
// 16*D bytes in its page), filled by 1-D bulk copies (cp.async.bulk, no
// multicast) that complete on a "full" mbarrier; with RBG > 1 an "empty"
// mbarrier counts the consumers before a stage is refilled.  The ring keeps
// streaming across portion boundaries.  At the end of a portion the streams
// combine their online-softmax states in shared memory; a segment held by one
// CTA is written out as bf16, otherwise the CTA writes (O/l, log2-sum-exp) to
// its part's slot and the CTA that finishes the segment last -- one atomic
// counter per segment, no waiting -- merges the parts and resets the counter.
// Every mbarrier wait is bounded (p.wait_limit_ns of wall clock, 200 ms by
// default): a wait that runs out flags ATLAS_DEVERR_TIMEOUT and the warp stops
// computing after draining its loads.
#include <float.h>
#include <math.h>

#include "atlas_internal.cuh"

namespace atlas {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kUnit = 32;  // tokens per pipeline unit (two 16-token pieces)
constexpr int kQBuf = 3;   // Q row buffers: portion pi + 2 loads while pi computes

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

// 16-byte global -> shared copy that completes asynchronously (cp.async, L2 only)
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_group1() {  // all but the newest group
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

// ----------------------------------------------------------- shared memory plan

// One portion: the part of segment (b, seg) that lies in this CTA's range.
struct Portion {
  int b, seg;           // sequence, segment within the sequence (h * row_blocks + rg)
  int L;                // the sequence's length
  int ua;               // first unit of the portion inside the segment
  int k0;               // first unit of the portion inside the CTA's range
  int slot0;            // first partial slot of the segment
  int my, n_parts;      // this portion's part index and the segment's part count
  int ql, qb;           // the sequence's new rows and its first packed q / out row
  float k_scale, v_scale;  // the KV head's dequantisation scales
};

// Dynamic shared memory: [ring][mbarriers][Q rows x kQBuf][combine][unit pieces]
// [portions].  Only 16-byte alignment is needed (bulk copies, cp.async,
// ldmatrix, vector loads).
struct SmemPlan {
  size_t bars, qbuf, combine, pieces, portions, total;
};
__host__ __device__ inline SmemPlan smem_plan(int D, int S, int nstream, int rows, int max_units,
                                              int max_portions) {
  SmemPlan sp;
  const size_t ring = (size_t)nstream * S * 4 * 16 * D;
  sp.bars = ring;
  sp.qbuf = sp.bars + (size_t)2 * nstream * S * 8;
  sp.combine = sp.qbuf + (size_t)kQBuf * rows * D * 2;
  // per stream and row: m and l (float), O / l (half)
  const size_t comb = nstream > 1 ? (size_t)nstream * rows * (8 + 2 * D) : 0;
  sp.pieces = sp.combine + (comb + 15) / 16 * 16;
  sp.portions = sp.pieces + (size_t)max_units * 8;
  sp.total = sp.portions + (size_t)max_portions * sizeof(Portion) + 16;
  return sp;
}

// Exclusive prefix sum of v over the CTA's threads (all threads call it);
// `total` receives the sum over the CTA.  `warp_sums` holds kWarps entries.
__device__ __forceinline__ unsigned long long block_exclusive_scan(unsigned long long v,
                                                                  unsigned long long* warp_sums,
                                                                  unsigned long long& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long x = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  unsigned long long base = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    if (w < warp) base += warp_sums[w];
    total += warp_sums[w];
  }
  __syncthreads();  // warp_sums may be reused
  return base + incl - v;
}

// CTA that owns global unit u under the balanced partition of U units over G CTAs
__device__ __forceinline__ int owner_cta(long long u, long long U, int G) {
  return (int)(((u + 1) * G - 1) / U);
}

// ------------------------------------------------------------------- the kernel

template <int D, int NT, int RBG, int S, bool PK>
__global__ void __launch_bounds__(kThreads, NT == 1 ? 3 : 2)
    paged_decode_fp8_kernel(const DecodeParams p) {
  // PK (packed): a warp holds 4 query rows, and the 8 columns of every MMA's N
  // side carry the hi parts (columns 0-3) and the lo parts (columns 4-7) of
  // those rows' Q (for QK^T) and P (for PV), so one MMA does the work of two
  static_assert(!PK || (NT == 1 && RBG == 1), "packed mode is 4 rows, one warp per stream");
  constexpr int RW = PK ? 4 : 8 * NT;    // query rows per warp
  constexpr int RC = RW * RBG;           // query rows per CTA
  constexpr int NSTREAM = kWarps / RBG;  // unit streams per CTA
  constexpr int NCH = D / 64;            // 16-byte K chunks per token per lane
  constexpr int KSTEP = D / 32;          // k-steps of QK^T
  constexpr int MT = D / 16;             // m-tiles of O^T
  constexpr int TILE = 16 * D;           // one 16-token K piece or V^T piece
  constexpr int STAGE = 4 * TILE;        // K_A, K_B, V_A, V_B

  const int Rmax = p.q_len * p.G;        // p.q_len: the largest q_len of any sequence
  const int rows_max = min(RC, Rmax);    // rows of the fullest row group
  extern __shared__ __align__(16) uint8_t smem[];
  const SmemPlan sp = smem_plan(D, S, NSTREAM, rows_max, p.max_units, p.max_portions);
  uint8_t* ring = smem;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + sp.bars);
  uint64_t* empty_bar = full_bar + NSTREAM * S;
  __nv_bfloat16* s_q = reinterpret_cast<__nv_bfloat16*>(smem + sp.qbuf);
  float* s_cm = reinterpret_cast<float*>(smem + sp.combine);  // [NSTREAM][rows_max]
  float* s_cl = s_cm + NSTREAM * rows_max;                      // [NSTREAM][rows_max]
  __half* s_co = reinterpret_cast<__half*>(s_cl + NSTREAM * rows_max);  // [NSTREAM][rows_max][D]
  int2* s_pieces = reinterpret_cast<int2*>(smem + sp.pieces);
  Portion* s_port = reinterpret_cast<Portion*>(smem + sp.portions);
  __shared__ int s_is_last;
  __shared__ int s_nport;
  __shared__ unsigned long long s_scan[kWarps];
  __shared__ float s_rowM[RC], s_rowD[RC];

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, c = lane & 3;
  const int stream = warp / RBG, rbw = warp % RBG;
  const int cid = blockIdx.x, G = gridDim.x;
  const int RB = p.row_blocks;          // row groups per (b, h)
  const int Hs = p.Hkv * RB;            // segments per sequence
  // new rows of sequence b and its first row in q / out: uniform q_len, or
  // per sequence from the packed offsets cu_q (ragged verify, prefill chunks)
  auto qlen_of = [&](int b) {
    return p.cu_q ? __ldg(p.cu_q + b + 1) - __ldg(p.cu_q + b) : p.q_len;
  };
  auto qbase_of = [&](int b) { return p.cu_q ? __ldg(p.cu_q + b) : b * p.q_len; };
  // a sequence with rows is served when q_len <= L <= the table row and the
  // host's max_seq_len; one with no rows (ragged only) is skipped silently
  auto valid_len = [&](int L, int ql) {
    return ql >= 1 && L >= ql && L <= p.max_blocks * p.ps && L <= p.max_seq_len;
  };
  auto units_of = [&](int L) { return (L + kUnit - 1) / kUnit; };

  // ---- invalid sequences (shorter than q_len, longer than the block-table row
  // or the host's max_seq_len): zero all their rows and flag them; one CTA per b
  for (int bb = cid; bb < p.B; bb += G) {
    const int L = __ldg(p.seq_lens + bb);
    const int ql = qlen_of(bb);
    if (ql == 0 || valid_len(L, ql)) continue;
    if (tid == 0) atomicOr(p.err, ATLAS_DEVERR_SEQ_LEN);
    const size_t n = (size_t)max(ql, 0) * p.Hq * D;
    __nv_bfloat16* o = p.out + (size_t)qbase_of(bb) * p.Hq * D;
    for (size_t idx = tid; idx < n; idx += kThreads) o[idx] = __float2bfloat16_rn(0.f);
  }

  // ---- this CTA's range of units and its portions (A1)
  long long u0 = 0, u1 = 0;
  if (p.grid_mode) {
    // CTA cid is split (cid % num_splits) of segment (cid / num_splits): tokens
    // [split * T, split * T + T) of it, one portion; a sequence split in n_parts
    // leaves n_parts partials (slots segment * num_splits + split).  Segment-
    // major order (the splits of a segment are neighbours) measured 2.5 % faster
    // than split-major on the LLaMA-shaped and long-context workloads, and
    // faster than the tensor-core kernel's longest-first order on both (44.7
    // vs 47.8 and 143.2 vs 148.3 µs): with three CTAs per SM the first wave
    // holds nearly all of the LLaMA-shaped launch, and the hardware deals it
    // to the SMs round-robin, so a sorted order gives some SMs only whole
    // splits and others only the short second ones.
    const int split = cid % p.num_splits, sg = cid / p.num_splits;
    const int b = sg / Hs, seg = sg % Hs;
    const int L = __ldg(p.seq_lens + b);
    const int ql = qlen_of(b);
    if (!valid_len(L, ql)) return;  // CTA-uniform; its rows were zeroed above
    if ((seg % RB) * RC >= ql * p.G) return;  // a row block past this sequence's rows
    const int t_begin = split * p.split_tokens;
    if (t_begin >= L) return;
    if (tid == 0) {
      Portion P;
      P.b = b; P.seg = seg; P.L = L; P.ua = t_begin / kUnit; P.k0 = 0;
      P.ql = ql; P.qb = qbase_of(b);
      P.slot0 = sg * p.num_splits;
      P.my = split;
      P.n_parts = (L + p.split_tokens - 1) / p.split_tokens;
      P.k_scale = __ldg(p.k_scale + seg / RB);
      P.v_scale = __ldg(p.v_scale + seg / RB);
      s_port[0] = P;
      s_nport = 1;
    }
    u1 = units_of(min(L - t_begin, p.split_tokens));
  } else {
    // every thread takes a contiguous run of sequences; a block-wide exclusive
    // scan of the runs' unit counts gives each run's first global unit
    const int per = (p.B + kThreads - 1) / kThreads;
    const int bb0 = min(p.B, tid * per), bb1 = min(p.B, bb0 + per);
    unsigned long long mine = 0;
    for (int bb = bb0; bb < bb1; ++bb) {
      const int L = __ldg(p.seq_lens + bb);
      if (valid_len(L, qlen_of(bb))) mine += (unsigned long long)Hs * units_of(L);
    }
    unsigned long long total = 0;
    const unsigned long long first = block_exclusive_scan(mine, s_scan, total);
    const long long U = (long long)total;
    // with fewer units than CTAs only the first U CTAs take one unit each, so
    // that every CTA between the first and last owner of a segment holds part
    // of it (the merge counts on that)
    const int Ge = (int)min((long long)G, U);
    if (cid >= Ge) return;  // CTA-uniform from here on (U == 0 included)
    u0 = (long long)((unsigned long long)cid * total / Ge);
    u1 = (long long)((unsigned long long)(cid + 1) * total / Ge);
    if (u1 - u0 > p.max_units) {  // only if a length exceeded the host's bound
      if (tid == 0) atomicOr(p.err, ATLAS_DEVERR_SEQ_LEN);
      return;
    }
    // portions: the segments of this thread's sequences that meet [u0, u1),
    // counted, scanned and written in list order (no sorting needed)
    int n_mine = 0;
    {
      long long P = (long long)first;
      for (int bb = bb0; bb < bb1 && P < u1; ++bb) {
        const int L = __ldg(p.seq_lens + bb);
        if (!valid_len(L, qlen_of(bb))) continue;
        const int n = units_of(L);
        const long long size = (long long)Hs * n;
        if (P + size > u0) {
          const long long s_lo = max(u0 - P, 0LL) / n;
          const long long s_hi = (min(u1, P + size) - 1 - P) / n;
          n_mine += (int)(s_hi - s_lo + 1);
        }
        P += size;
      }
    }
    unsigned long long n_all = 0;
    int slot_out = (int)block_exclusive_scan((unsigned long long)n_mine, s_scan, n_all);
    if (tid == 0) s_nport = (int)n_all;
    {
      long long P = (long long)first;
      for (int bb = bb0; bb < bb1 && P < u1; ++bb) {
        const int L = __ldg(p.seq_lens + bb);
        if (!valid_len(L, qlen_of(bb))) continue;
        const int n = units_of(L);
        const long long size = (long long)Hs * n;
        if (P + size > u0) {
          const int s_lo = (int)(max(u0 - P, 0LL) / n);
          const int s_hi = (int)((min(u1, P + size) - 1 - P) / n);
          for (int seg = s_lo; seg <= s_hi; ++seg) {
            const long long s0 = P + (long long)seg * n;
            const long long a = max(s0, u0);
            Portion Q;
            Q.b = bb; Q.seg = seg; Q.L = L;
            Q.ql = qlen_of(bb); Q.qb = qbase_of(bb);
            Q.ua = (int)(a - s0);
            Q.k0 = (int)(a - u0);
            const int c_first = owner_cta(s0, U, Ge);
            Q.slot0 = (bb * Hs + seg) + c_first;
            Q.my = cid - c_first;
            Q.n_parts = owner_cta(s0 + n - 1, U, Ge) - c_first + 1;
            Q.k_scale = __ldg(p.k_scale + seg / RB);
            Q.v_scale = __ldg(p.v_scale + seg / RB);
            s_port[slot_out++] = Q;
          }
        }
        P += size;
      }
    }
  }
  __syncthreads();
  const int n_port = s_nport;
  const int U_cta = (int)(u1 - u0);
  // portion p covers CTA units [k0_p, k0_{p+1})
  auto port_end = [&](int pi) { return pi + 1 < n_port ? s_port[pi + 1].k0 : U_cta; };

  // Q rows of portion pi -> Q buffer pi % kQBuf, one cp.async group per call
  auto prefetch_q = [&](int pi) {
    const Portion P = s_port[pi];
    const int h = P.seg / RB, r0 = (P.seg % RB) * RC;
    const int rows = max(0, min(RC, P.ql * p.G - r0));
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    __nv_bfloat16* dst = s_q + (size_t)(pi % kQBuf) * rows_max * D;
    for (int idx = tid; idx < rows * CPR; idx += kThreads) {
      const int lr = idx / CPR, ch = idx - lr * CPR;
      const int r = r0 + lr;
      const int i = r / p.G, hq = h * p.G + r % p.G;
      cp_async16(dst + lr * D + ch * 8,
                 p.q + (((size_t)P.qb + i) * p.Hq + hq) * D + ch * 8);
    }
    cp_async_commit();
  };
  prefetch_q(0);
  if (n_port > 1) prefetch_q(1);

  // ---- A2, block-table gather: the two 16-token pieces of unit k of the
  // range, as indices of 16*D-byte blocks of the page arrays (-1: past the end
  // of the sequence or a bad page id).  The divisions happen here, once.
  const int groups_per_page = p.ps / 16;
  auto build_piece = [&](int k) {
    int lo = 0, hi = n_port - 1;   // last portion with k0 <= k
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_port[mid].k0 <= k) lo = mid; else hi = mid - 1;
    }
    const Portion P = s_port[lo];
    const int h = P.seg / RB;
    const int t0 = kUnit * (P.ua + k - P.k0);
    int pc[2];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int t = t0 + 16 * half;
      pc[half] = -1;
      if (t < P.L) {
        const int pg = t / p.ps;
        const int pid = __ldg(p.block_table + (size_t)P.b * p.max_blocks + pg);
        if (pid < 0 || pid >= p.num_pages)
          atomicOr(p.err, ATLAS_DEVERR_PAGE_ID);
        else
          pc[half] = (pid * p.Hkv + h) * groups_per_page + (t - pg * p.ps) / 16;
      }
    }
    s_pieces[k] = make_int2(pc[0], pc[1]);
  };
  // ---- A0, fused append: the step's new tokens (positions L - q_len .. L - 1)
  // that fall in this CTA's portions are quantised and stored first, while HBM
  // is still idle, and made visible to the bulk copies before any is queued
  if (p.k_new != nullptr) {
    bool wrote = false;
    for (int pi = 0; pi < n_port; ++pi) {
      const Portion P = s_port[pi];
      const int L = P.L;
      const int h = P.seg / RB;
      const int first_new_pos = L - P.ql;
      const int a0 = max(kUnit * P.ua, first_new_pos);
      const int a1 = min(kUnit * (P.ua + port_end(pi) - P.k0), L);
      const int n_tok = a1 - a0;
      if (n_tok <= 0) continue;
      wrote = true;
      constexpr int CH = D / 16;
      for (int idx = tid; idx < 2 * n_tok * CH; idx += kThreads) {
        const int which = idx / (n_tok * CH);  // 0 = K, 1 = V
        const int r = idx - which * n_tok * CH;
        const int pos = a0 + r / CH, j = r % CH;
        const int page = __ldg(p.block_table + (size_t)P.b * p.max_blocks + pos / p.ps);
        if (page < 0 || page >= p.num_pages) {
          atomicOr(p.err, ATLAS_DEVERR_APPEND);
          continue;
        }
        float x[16];
        load16_as_f32(which ? p.v_new : p.k_new,
                      (((size_t)P.qb + (pos - first_new_pos)) * p.Hkv + h) * D + 16 * j,
                      p.new_dtype, x);
        const uint4 codes = quantize16_e4m3(x, which ? P.v_scale : P.k_scale);
        const size_t head_page = (size_t)page * p.Hkv + h;
        if (!which)
          store16_k(const_cast<uint8_t*>(p.k_pages), head_page, D, p.ps, pos % p.ps, j, codes);
        else
          store16_v(const_cast<uint8_t*>(p.v_pages), head_page, D, p.ps, pos % p.ps, j, codes);
      }
    }
    if (wrote) {
      __threadfence();
      fence_proxy_async_global();
    }
  }
  // the whole unit table, before any bulk copy is queued
  for (int k = tid; k < U_cta; k += kThreads) build_piece(k);
  if (tid < NSTREAM * S) {
    mbar_init(&full_bar[tid], 1);
    mbar_init(&empty_bar[tid], RBG);
  }
  if (tid == 0) fence_mbar_init();
  __syncthreads();  // table, barriers and appended tokens ready

  // this stream's units: k = stream + NSTREAM * i, i < n_my
  const int n_my = (stream < U_cta) ? (U_cta - stream + NSTREAM - 1) / NSTREAM : 0;
  const bool producer = (rbw == 0) && (lane == 0);
  constexpr size_t kPiece = (size_t)16 * D;  // bytes of one 16-token piece
  auto issue = [&](int i) {  // producer lane only: stage i % S <- unit i
    const int st = i % S;
    uint64_t* bar = &full_bar[stream * S + st];
    uint8_t* dst = ring + (size_t)(stream * S + st) * STAGE;
    if (p.test_skip_unit == i && cid == 0 && stream == 0) return;  // lost copy (tests only)
    const int2 pc = s_pieces[stream + NSTREAM * i];
    const uint32_t bytes = (pc.x >= 0 ? 2 * TILE : 0) + (pc.y >= 0 ? 2 * TILE : 0);
    if (bytes == 0) {
      mbar_arrive(bar);
      return;
    }
    mbar_arrive_expect_tx(bar, bytes);
    // a 16-token piece is TILE contiguous bytes in both layouts: K rows
    // (slot0 .. slot0 + 15) x D, and V group slot0 / 16 ([D][16])
    if (pc.x >= 0) {
      bulk_load(dst, p.k_pages + (size_t)pc.x * kPiece, TILE, bar);
      bulk_load(dst + 2 * TILE, p.v_pages + (size_t)pc.x * kPiece, TILE, bar);
    }
    if (pc.y >= 0) {
      bulk_load(dst + TILE, p.k_pages + (size_t)pc.y * kPiece, TILE, bar);
      bulk_load(dst + 3 * TILE, p.v_pages + (size_t)pc.y * kPiece, TILE, bar);
    }
  };
  if (producer) {
    for (int i = 0; i < S && i < n_my; ++i) issue(i);
  }


  // per-portion state (re-initialised for every portion)
  uint32_t qhi[NT][KSTEP][2], qlo[NT][KSTEP][2];
  int lim[NT][2];
  float scale2[NT][2];
  int min_lim = 0;
  float m_run[NT][2], l_run[NT][2];
  float acc[MT][NT][4];

  // this lane's K operand words of one 16-token K tile: rows g8 and g8 + 8,
  // 16-byte chunks 4j + c.  D = 128: the pages store chunk j of slot s at
  // j XOR (s % 8), and a 16-token piece starts at a multiple of 16 slots, so
  // row g8 (+ 8) finds logical chunk 4j + c at (4j + c) ^ g8 -- which also
  // puts the 8 lanes of each shared-memory phase on distinct banks
  auto load_k = [&](const uint8_t* kt, uint4 (&kr)[2][NCH]) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int row = g8 + 8 * t;
      if constexpr (D == 128) {
        const uint8_t* rb = kt + row * 128;
        kr[t][0] = *reinterpret_cast<const uint4*>(rb + (((0 + c) ^ g8) << 4));
        kr[t][1] = *reinterpret_cast<const uint4*>(rb + (((4 + c) ^ g8) << 4));
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
          if constexpr (PK) {
            // packed hi | lo columns; even and odd k-steps go to separate
            // accumulators so that four chains still interleave
            if (hs == 0) {
              mma_e4m3(ah[nt], a0, a1, a2, a3, qhi[nt][ks][0], qhi[nt][ks][1]);
              mma_e4m3(bh[nt], c0, c1, c2, c3, qhi[nt][ks][0], qhi[nt][ks][1]);
            } else {
              mma_e4m3(al[nt], a0, a1, a2, a3, qhi[nt][ks][0], qhi[nt][ks][1]);
              mma_e4m3(bl[nt], c0, c1, c2, c3, qhi[nt][ks][0], qhi[nt][ks][1]);
            }
          } else {
            mma_e4m3(ah[nt], a0, a1, a2, a3, qhi[nt][ks][0], qhi[nt][ks][1]);
            mma_e4m3(bh[nt], c0, c1, c2, c3, qhi[nt][ks][0], qhi[nt][ks][1]);
            mma_e4m3(al[nt], a0, a1, a2, a3, qlo[nt][ks][0], qlo[nt][ks][1]);
            mma_e4m3(bl[nt], c0, c1, c2, c3, qlo[nt][ks][0], qlo[nt][ks][1]);
          }
        }
      }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        sa[nt][e] = ah[nt][e] + al[nt][e];
        sb[nt][e] = bh[nt][e] + bl[nt][e];
        if constexpr (PK) {  // column 2c + e holds hi, column 2c + e ^ 4 lo: add them
          sa[nt][e] += __shfl_xor_sync(kFull, sa[nt][e], 2);
          sb[nt][e] += __shfl_xor_sync(kFull, sb[nt][e], 2);
        }
      }
  };

  auto compute_unit = [&](int t0, int nvA, int nvB, const uint8_t* stage) {
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
      if constexpr (PK) {  // B columns 0-3: hi parts, 4-7: lo parts of the same rows
        if (g8 >= 4) {
          pbhi[nt][0] = pblo[nt][0];
          pbhi[nt][1] = pblo[nt][1];
        }
      }
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
        if constexpr (!PK) mma_e4m3(acc[mt][nt], a0, a1, a2, a3, pblo[nt][0], pblo[nt][1]);
      }
    }
  };

  int i_next = 0;  // next stream-local unit to consume
  bool aborted = false;
  int n_cut = 0, cut0 = 0, cut1 = 0;  // portions whose segment other CTAs share (<= 2)
#pragma unroll 1
  for (int pi = 0; pi < n_port; ++pi) {
    const Portion P = s_port[pi];
    const int seg = P.seg, L = P.L;
    const int h = seg / RB, rg = seg % RB;
    const int Rtot = P.ql * p.G;           // this sequence's query rows per KV head
    const int cta_row0 = rg * RC;
    const int rows_cta = max(0, min(RC, Rtot - cta_row0));
    const int row0 = cta_row0 + rbw * RW;  // this warp's first row
    const int kb = P.k0, ke = port_end(pi);
    const bool whole = (P.n_parts == 1);
    if (!whole) {
      if (n_cut == 0) cut0 = pi; else cut1 = pi;
      n_cut = min(n_cut + 1, 2);
    }

    // groups in flight: portions pi and (if it exists) pi + 1; wait for pi's
    if (pi + 1 < n_port) cp_async_wait_group1(); else cp_async_wait_all();
    __syncthreads();  // this portion's Q rows are in buffer pi % kQBuf
    if (pi + 2 < n_port) prefetch_q(pi + 2);  // into the buffer portion pi - 1 used
    const __nv_bfloat16* qb = s_q + (size_t)(pi % kQBuf) * rows_max * D;

    // ---- Q^T fragments as E4M3 hi + lo with a per-row power-of-two scale
    // B operand of k-step s = 2j + hs: b0 = dims 64j+16c+8hs+{0..3}, b1 = +{4..7}.
    float alpha_row[NT];  // the scale of row 8nt + g8
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      // row within the row group (PK: lanes g8 and g8 + 4 both prepare row g8 % 4)
      const int lr = PK ? (g8 & 3) : rbw * RW + 8 * nt + g8;
      float x[NCH][16];
      if (cta_row0 + lr < Rtot) {
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
          const uint4* src = reinterpret_cast<const uint4*>(qb + lr * D + j * 64 + 16 * c);
          const uint4 w0 = src[0], w1 = src[1];
          const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
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
            // PK: lanes g8 < 4 feed the hi columns, lanes g8 >= 4 the lo columns
            qhi[nt][2 * j + hs][half] = (PK && g8 >= 4) ? (l01 | (l23 << 16)) : (h01 | (h23 << 16));
            qlo[nt][2 * j + hs][half] = l01 | (l23 << 16);
          }
    }
    // per accumulator row (8nt + 2c + e): causal limit and score scale
    const float kscale = P.k_scale * p.qk_scale_log2;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        // the row of accumulator column 2c + e (PK: columns c and c ^ 2 are one row)
        const int rl = PK ? 2 * (c & 1) + e : 8 * nt + 2 * c + e;
        const int r = row0 + rl;
        lim[nt][e] = (r < Rtot) ? (L - P.ql + r / p.G) : (L - 1);
        const float a = __shfl_sync(kFull, alpha_row[nt], 4 * (rl - 8 * nt));
        scale2[nt][e] = kscale / a;
      }
    min_lim = L - P.ql + row0 / p.G;
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

    // ---- this stream's units of the portion: k in [kb, ke), k = stream + NSTREAM*i
#pragma unroll 1
    for (; !aborted; ++i_next) {
      const int k = stream + NSTREAM * i_next;
      if (k >= ke) break;
      const int st = i_next % S;
      const uint32_t par = (uint32_t)((i_next / S) & 1);
      if (!mbar_wait_bounded(&full_bar[stream * S + st], par, p.wait_limit_ns)) {
        aborted = true;
        break;
      }
      if (row0 < Rtot) {
        const int2 pc = s_pieces[k];
        const int t0 = kUnit * (P.ua + k - kb);
        const int nvA = pc.x >= 0 ? min(16, L - t0) : 0;
        const int nvB = pc.y >= 0 ? min(16, L - t0 - 16) : 0;
        compute_unit(t0, nvA, nvB, ring + (size_t)(stream * S + st) * STAGE);
      }
      __syncwarp();
      if constexpr (RBG > 1) {
        if (lane == 0) mbar_arrive(&empty_bar[stream * S + st]);
      }
      if (producer && i_next + S < n_my) {
        if constexpr (RBG > 1) {
          if (!mbar_wait_bounded(&empty_bar[stream * S + st], par, p.wait_limit_ns)) aborted = true;
        }
        // the stage's readers are done: RBG = 1, their loads fed this warp's MMAs
        // before the __syncwarp; RBG > 1, the empty barrier ordered them
        if (!aborted) issue(i_next + S);
      }
      if (__any_sync(kFull, aborted)) aborted = true;
    }

    // ---- PK: O's hi and lo columns (lanes c and c ^ 2) add up to the row's O
    if constexpr (PK) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][0][e] += __shfl_xor_sync(kFull, acc[mt][0][e], 2);
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

    // ---- where the portion's result goes: the output, or the partial slot of
    // this part when other CTAs hold the segment's other parts
    const float vs = P.v_scale;
    const size_t slot = (size_t)P.slot0 + P.my;

    if constexpr (NSTREAM == 1) {
      // one stream: every warp owns its rows outright; store from registers
      if (row0 < Rtot) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int lr = rbw * RW + 8 * nt + 2 * c + e;
            const int r = cta_row0 + lr;
            if (r >= Rtot) continue;
            const int i = r / p.G, hq = h * p.G + r % p.G;
            const float den = l_full[nt][e];
            const float inv = den > 0.f ? 1.f / den : 0.f;
            if (whole) {
              __nv_bfloat16* orow = p.out + (((size_t)P.qb + i) * p.Hq + hq) * D;
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) {
                orow[16 * mt + g8] = __float2bfloat16_rn(acc[mt][nt][e] * inv * vs);
                orow[16 * mt + g8 + 8] = __float2bfloat16_rn(acc[mt][nt][e + 2] * inv * vs);
              }
            } else {
              float* prow = p.part_o + (slot * RC + lr) * D;
#pragma unroll
              for (int mt = 0; mt < MT; ++mt) {
                prow[16 * mt + g8] = acc[mt][nt][e] * inv;
                prow[16 * mt + g8 + 8] = acc[mt][nt][e + 2] * inv;
              }
              if (g8 == 0)
                p.part_lse[slot * RC + lr] = den > 0.f ? m_run[nt][e] + __log2f(den) : -INFINITY;
            }
          }
      }
    } else {
      // streams leave (m, l, O / l) of their rows in shared memory; all
      // threads combine them (O / l is at most max|v| <= 448: half is enough)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int lr = PK ? 2 * c + e : rbw * RW + 8 * nt + 2 * c + e;
          if (lr < rows_cta && (!PK || c < 2)) {
            const float den = l_full[nt][e];
            const float inv = den > 0.f ? 1.f / den : 0.f;
            if (g8 == 0) {
              s_cm[stream * rows_max + lr] = m_run[nt][e];
              s_cl[stream * rows_max + lr] = den;
            }
            __half* orow = s_co + ((size_t)stream * rows_max + lr) * D;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              orow[16 * mt + g8] = __float2half_rn(acc[mt][nt][e] * inv);
              orow[16 * mt + g8 + 8] = __float2half_rn(acc[mt][nt][e + 2] * inv);
            }
          }
        }
      __syncthreads();
      for (int idx = tid; idx < rows_cta * D; idx += kThreads) {
        const int lr = idx / D, d = idx - lr * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NSTREAM; ++w) M = fmaxf(M, s_cm[w * rows_max + lr]);
        float den = 0.f, num = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < NSTREAM; ++w) {
            const float f = fast_exp2(s_cm[w * rows_max + lr] - M) * s_cl[w * rows_max + lr];
            den += f;
            num += f * __half2float(s_co[((size_t)w * rows_max + lr) * D + d]);
          }
        }
        const int r = cta_row0 + lr;
        const int i = r / p.G, hq = h * p.G + r % p.G;
        if (whole) {
          p.out[(((size_t)P.qb + i) * p.Hq + hq) * D + d] =
              __float2bfloat16_rn(den > 0.f ? num / den * vs : 0.f);
        } else {
          p.part_o[(slot * RC + lr) * D + d] = (den > 0.f) ? num / den : 0.f;
          // the log2-sum-exp carries the 2^8 factor of p; it cancels in the merge
          if (d == 0) p.part_lse[slot * RC + lr] = (den > 0.f) ? M + __log2f(den) : -INFINITY;
        }
      }
    }
    // the combine buffer is free for the next portion; a timeout anywhere stops the CTA
    if (__syncthreads_or(aborted)) {
      aborted = true;
      break;
    }
  }

  if (aborted) {
    if (lane == 0) atomicOr(p.err, ATLAS_DEVERR_TIMEOUT);
    // drain this stream's loads still in flight (issued: i < min(n_my, i_next + S))
    for (int i = i_next; i < n_my && i < i_next + S; ++i)
      mbar_wait_bounded(&full_bar[stream * S + i % S], (uint32_t)((i / S) & 1), p.wait_limit_ns);
    cp_async_wait_all();
    return;
  }
  if (n_cut == 0) return;

  // ---- segments shared with other CTAs (A8 -> A9): one completion counter per
  // segment; the CTA that finishes a segment last merges its partial slots.
  // Done once at the end, so that no portion waits on a fence or an atomic.
  __threadfence();
  for (int q = 0; q < n_cut; ++q) {
    const Portion P = s_port[q == 0 ? cut0 : cut1];
    const int seg_idx = P.b * Hs + P.seg;
    const int h = P.seg / RB, cta_row0 = (P.seg % RB) * RC;
    const int rows_cta = max(0, min(RC, P.ql * p.G - cta_row0));
    int32_t* counter = p.counters + seg_idx;
    __syncthreads();  // every thread's partial stores are fenced; s_is_last is free
    if (tid == 0) s_is_last = (atomicAdd(counter, 1) == P.n_parts - 1);
    __syncthreads();
    if (!s_is_last) continue;
    __threadfence();
    const size_t s0 = (size_t)P.slot0;
    const int n_slots = P.n_parts;
    // per row: reference M and denominator over the slots' log2-sum-exp values
    for (int lr = tid; lr < rows_cta; lr += kThreads) {
      float M = -INFINITY, den = 0.f;
      for (int sl = 0; sl < n_slots; ++sl) {
        const float v = __ldcg(p.part_lse + (s0 + sl) * RC + lr);
        if (v == -INFINITY) continue;
        if (v > M) {
          den = den * fast_exp2(M - v) + 1.f;
          M = v;
        } else {
          den += fast_exp2(v - M);
        }
      }
      s_rowM[lr] = M;
      s_rowD[lr] = den;
    }
    __syncthreads();
    const float vs = P.v_scale;
    constexpr int C4 = D / 4;
    for (int idx = tid; idx < rows_cta * C4; idx += kThreads) {
      const int lr = idx / C4, d0 = 4 * (idx - lr * C4);
      const float M = s_rowM[lr], den = s_rowD[lr];
      float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
      if (den > 0.f) {
#pragma unroll 4
        for (int sl = 0; sl < n_slots; ++sl) {
          const float wgt = fast_exp2(__ldcg(p.part_lse + (s0 + sl) * RC + lr) - M);
          const float4 v =
              __ldcg(reinterpret_cast<const float4*>(p.part_o + ((s0 + sl) * RC + lr) * D + d0));
          o4.x += wgt * v.x; o4.y += wgt * v.y; o4.z += wgt * v.z; o4.w += wgt * v.w;
        }
      }
      const float inv = den > 0.f ? vs / den : 0.f;
      const int r = cta_row0 + lr;
      const int i = r / p.G, hq = h * p.G + r % p.G;
      __nv_bfloat16* dst = p.out + (((size_t)P.qb + i) * p.Hq + hq) * D + d0;
      const __nv_bfloat162 lo = __floats2bfloat162_rn(o4.x * inv, o4.y * inv);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(o4.z * inv, o4.w * inv);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t*>(&lo);
      pk.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(dst) = pk;
    }
    if (tid == 0) *counter = 0;  // ready for the next call on this stream
  }
}

// ------------------------------------------------------------------- launching

template <int D, int NT, int RBG, int S, bool PK>
struct Cfg {
  static constexpr auto kernel() { return paged_decode_fp8_kernel<D, NT, RBG, S, PK>; }
};

// Calls f(Cfg<...>{}) for the instantiation that serves these parameters.
template <int D, int NT, int RBG, bool PK, class F>
cudaError_t with_stages(int stages, F&& f) {
  if (stages == 2) return f(Cfg<D, NT, RBG, 2, PK>{});
  if (stages == 3) return f(Cfg<D, NT, RBG, 3, PK>{});
  return cudaErrorInvalidValue;
}
template <int D, class F>
cudaError_t with_rows(int rows_per_warp, int rbg, int stages, F&& f) {
  if (rows_per_warp == 4 && rbg == 1) return with_stages<D, 1, 1, true>(stages, f);
  if (rows_per_warp == 8 && rbg == 1) return with_stages<D, 1, 1, false>(stages, f);
  if (rows_per_warp == 16 && rbg == 1) return with_stages<D, 2, 1, false>(stages, f);
  if (rows_per_warp == 16 && rbg == 2) return with_stages<D, 2, 2, false>(stages, f);
  if (rows_per_warp == 16 && rbg == 4) return with_stages<D, 2, 4, false>(stages, f);
  return cudaErrorInvalidValue;
}
template <class F>
cudaError_t with_kernel(int D, int rows_per_warp, int rbg, int stages, F&& f) {
  if (D == 128) return with_rows<128>(rows_per_warp, rbg, stages, f);
  if (D == 64) return with_rows<64>(rows_per_warp, rbg, stages, f);
  return cudaErrorInvalidValue;
}

}  // namespace

size_t decode_fp8_smem_bytes(int D, int stages, int rbg, int rows, int max_units,
                             int max_portions) {
  return smem_plan(D, stages, kWarps / rbg, rows, max_units, max_portions).total;
}

void decode_fp8_fit_grid(int D, int rows, int sms, DecodeLaunch& L) {
  if (L.grid_mode) return;
  for (int it = 0; it < 4; ++it) {
    const size_t smem = decode_fp8_smem_bytes(D, L.stages, L.rbg, rows, L.max_units,
                                              L.max_portions);
    int occ = 0;
    const cudaError_t e = with_kernel(D, L.rows_per_warp, L.rbg, L.stages, [&](auto cfg) {
      auto kern = decltype(cfg)::kernel();
      cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (r != cudaSuccess) return r;
      return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, smem);
    });
    if (e != cudaSuccess || occ <= 0) {
      cudaGetLastError();
      return;  // the launch reports the problem
    }
    const long long resident = (long long)sms * occ * L.waves;
    if (L.grid <= resident) return;
    const long long mu = (L.units_max + resident - 1) / resident;
    if (mu > kMaxUnitsPerCta) return;
    L.grid = resident;
    L.max_units = (int)mu;
    L.max_portions = (int)(L.segs < mu ? L.segs : mu);
  }
}

cudaError_t launch_decode_fp8(const DecodeParams& p, int rows_per_warp, int rbg, int stages,
                              long long grid, cudaStream_t stream) {
  if (grid < 1 || grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const int rows = min(rows_per_warp * rbg, p.q_len * p.G);
  const size_t smem = decode_fp8_smem_bytes(p.D, stages, rbg, rows, p.max_units, p.max_portions);
  return with_kernel(p.D, rows_per_warp, rbg, stages, [&](auto cfg) {
    auto kern = decltype(cfg)::kernel();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
  });
}

}  // namespace atlas
