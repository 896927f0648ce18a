// Paged FP8 decode / MTP-verify grouped-query attention on the 5th-generation
// tensor cores (tcgen05.mma, accumulators in tensor memory), for KV heads
// whose q_len x G query rows fill a real contraction (the 27B-class MTP
// verify with 25 rows, the MQA decode with 64).
//
// Computes the same masked SDPA over the dequantised paged cache as the warp-
// MMA kernel (decode_fp8.cu):
//     s_t = sm_scale * k_scale[h] * q . code(K[t, h, :])
//     out = v_scale[h] * sum_t softmax(s)_t * code(V[t, h, :]),  t <= L - q_len + i
// (the FlashAttention-2-style online softmax and dedicated GQA/MQA kernels of
// the Atlas deep-dive, ainews.cool, "Attention" paragraph; FP8 with scale
// factors, "Quantisation" paragraph; the paged FP8 KV cache with MTP K = 4
// verify of the GB10 page, ainews.surl.tw).
//
// CTA = one split of one segment (sequence b, KV head h, block of up to 64
// query rows), as in the grid partition: split_tokens KV tokens in tiles of
// 128.  The CTAs take their items longest first: every CTA ranks the items
// by a length key from seq_lens (a histogram and two block scans) and takes
// the one its index names -- the sequences cut into several splits first,
// segment-major, then the single-split ones by their number of tiles, so the
// short ones fill the end of the launch and the indices past the last item
// (splits past a sequence's end) come last.  Six warps:
//   * warp 4 -- producer: 1-D bulk copies (cp.async.bulk, no multicast) of
//     the tile's eight 16-token K pieces and eight V pieces (pieces adjacent
//     in a page go as one copy, one lane per run) into a K ring and a V ring
//     of S stages each, completion on "full" mbarriers; a K stage is refilled
//     once the S product has read it, a V stage once the PV product has;
//   * warp 5, lane 0 -- MMA issuer: per tile
//       S[64 rows x 128 tok] = (Qhi + Qlo)[64 x 128 d] . K_tile^T
//     as two M=64, N=64 halves (tokens 0-63 into TMEM lanes 0-15 of each warp
//     quadrant, tokens 64-127 into lanes 16-31), then, once the softmax has
//     written P,
//       O[64 x 128 d] += (Phi + Plo)[64 x 128 tok] . V_tile
//     as two M=64, N=64 halves (dims 0-63 in lanes 0-15, 64-127 in lanes
//     16-31).  kind::f8f6f4, E4M3 x E4M3, f32 accumulation; the cached codes
//     are the B operands as they lie in the pages (K rows carry the 128-byte
//     swizzle, V pages are [d][16 slots] core matrices);
//   * warps 0-3 -- softmax (those holding at least one of the block's rows;
//     the others sit out): thread (warp w, lane l) owns query row
//     16 w + (l % 16) and tokens / head dims 64 (l / 16) .. + 63 of every tile,
//     reads its S columns with tcgen05.ld, masks, keeps the online-softmax
//     state (running reference m and sum l, per row), writes P as E4M3 hi + lo
//     parts into shared memory (the A operand of the PV MMA) and, when a row's
//     reference moves, rescales that row's O in tensor memory.
// Numerics are those of the warp-MMA kernel: Q rows scaled by a power of two
// into (224, 448] and split into exact E4M3 hi + lo parts; p = 2^(s - m + 8)
// rounded to f16 and split into hi + lo (8 significant bits); the reference
// m of a row moves only when a score exceeds it by more than 0.5 (so
// p <= 2^8.5 fits E4M3), decided per row; l sums the f32 p.
//
// A segment cut into several splits leaves (O / l, log2-sum-exp) partials;
// the CTA that finishes the segment last (one atomic counter per segment)
// merges them.  Every mbarrier wait is bounded by p.wait_limit_ns; a wait
// that runs out flags ATLAS_DEVERR_TIMEOUT, the other roles stop, copies and
// MMAs in flight are drained (bounded), tensor memory is freed and the CTA
// returns without writing its rows.
#include <float.h>
#include <math.h>

#include "atlas_internal.cuh"

namespace atlas {
namespace {

constexpr int kThreads = 192;              // warps 0-3 softmax, 4 producer, 5 MMA
constexpr int kRows = 64;                  // query rows per CTA (MMA M)
constexpr int kTile = 128;                 // KV tokens per pipeline tile
constexpr int kD = 128;                    // head dim
constexpr int kPiece = 16 * kD;            // one 16-token K or V piece: 2048 bytes
constexpr int kTileBytes = 8 * kPiece;     // K (or V) of one tile: 16 KB
constexpr int kOpBytes = kRows * kD;       // one E4M3 part of Q or P: 8 KB
constexpr int kVS = 2;                     // V ring stages (the K ring has KS)
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0;              // S double buffer: columns 0-63, 64-127
constexpr uint32_t kColO = 128;            // O: columns 128-191
constexpr uint32_t kColQ = 192;            // Q hi: 192-223, Q lo: 224-255 (A operand)
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr int kWarps = kThreads / 32;
constexpr int kSchedExtra = kWarps + 4;    // scan partials + (bin, rank, b, split)

// ---------------------------------------------------------------- tcgen05 PTX

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(dst_smem)), "r"(cols) : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (tensor core, bulk copy) accesses.
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// D[tmem] (+)= A[smem] . B[smem]^T, kind::f8f6f4 (E4M3 x E4M3 -> f32).
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] . B[smem]^T, kind::f8f6f4, A read from tensor memory.
// With M = 64, row m of A sits in the same lane as row m of D (lanes 0-15 of
// each 32-lane quadrant, or 16-31 at lane offset 16), its K = 32 E4M3 values
// in 8 consecutive 32-bit columns, 4 per column in byte order.
__device__ __forceinline__ void mma_f8_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The mbarrier's phase completes once every tcgen05 operation this thread
// issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}

// Load 32 consecutive 32-bit columns of this thread's TMEM lane (32x32b
// shape: the warp reads the 32 lanes of its quadrant, lane id = lane), and
// wait for the load in the same statement so that no use of r can be
// scheduled before the data is there.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// Store 32 consecutive 32-bit columns of this thread's TMEM lane and wait for
// the store.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};\n\t"
      "tcgen05.wait::st.sync.aligned;"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
        "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
        "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Shared-memory matrix descriptor of a tcgen05 operand: start address, the
// leading- and stride-dimension byte offsets (16-byte units), the sm_100
// descriptor version (bit 46) and the swizzle mode (bits 61-63: 0 none,
// 2 = 128-byte).  Canonical K-major layouts: without swizzle, 8-row x 16-byte
// core matrices stored contiguously, LBO = distance between core matrices
// along K, SBO = along M/N; with the 128-byte swizzle, 128-byte rows in
// 1024-byte atoms of 8 rows, SBO = distance between atoms.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t swizzle) {
  uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)swizzle << 61;
  return d;
}

// Instruction descriptor, kind::f8f6f4: f32 accumulator (bits 4-5 = 1), A and
// B E4M3 (formats 0), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_f8(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------ helpers

__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t f16x2_to_e4m3x2(uint32_t x) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(r) : "r"(x));
  return r;
}
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
// Two probabilities -> N E4M3 pairs: f16 rounding, then part k = E4M3 of what
// the earlier parts leave (each subtraction is exact in f16).  Two parts
// carry 8 significant bits, three carry the f16 value's 11.
template <int N>
__device__ __forceinline__ void split_pair(float a, float b, uint32_t (&part)[N]) {
  uint32_t x = pack_f16x2(a, b);
#pragma unroll
  for (int k = 0; k < N; ++k) {
    part[k] = f16x2_to_e4m3x2(x);
    if (k + 1 < N) x = hsub2(x, e4m3x2_to_f16x2(part[k]));
  }
}

// Byte of slot t inside a 16-slot V group row: bytes 4c..4c+3 hold slots
// 2c, 2c+1, 2c+8, 2c+9.
__device__ __forceinline__ int group_pos(int t) {
  return 4 * ((t & 7) >> 1) + 2 * (t >> 3) + (t & 1);
}

// One probe of an mbarrier phase without a suspend-time hint: the hand-offs
// between the roles are short, and a thread put to sleep wakes up late.
__device__ __forceinline__ bool mbar_probe(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of an mbarrier phase (for the MMA issuer's event loop,
// which polls two conditions and must not be parked on either).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait that also gives up when another role has flagged an abort;
// a wait that runs out raises the abort flag.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                        uint64_t limit_cycles) {
  if (mbar_probe(bar, parity)) return true;
  const uint64_t t0 = sm_cycles();
  while (true) {
    if (mbar_probe(bar, parity)) return true;
    if (*abort_flag) return false;
    if (sm_cycles() - t0 > limit_cycles) {
      *abort_flag = 1;
      return false;
    }
  }
}

// ----------------------------------------------------------- shared memory

struct TcLayout {
  size_t k, v, ts, p, tab, sched, bar, misc, rows, total;
};
// E4M3 parts that carry a probability into the PV product: hi + lo (8
// significant bits); three with per-token V scales, where even the row's
// largest probability is no longer a power of two
__host__ __device__ constexpr int p_parts(bool tok_scales) { return tok_scales ? 3 : 2; }
// barriers: K ring full / empty / scales-read (KS each), V ring full / empty
// (kVS each), S buffers full / free (2 each), P full, PV done, drain, Q ready
__host__ __device__ constexpr int tc_barriers(int k_stages) { return 3 * k_stages + 2 * kVS + 8; }
// ts: per-token K scales of each K stage and V scales of each V stage
// (finer-grained mode), else empty
__host__ __device__ inline TcLayout tc_layout(int k_stages, int max_pieces, bool tok_scales) {
  TcLayout t;
  t.k = 0;                                              // [KS][8 pieces][16 tok][128 B] (swizzled)
  t.v = t.k + (size_t)k_stages * kTileBytes;            // [kVS][8 pieces][128 d][16 slots]
  t.ts = t.v + (size_t)kVS * kTileBytes;                // [KS][128] K scales, [kVS][128] V scales
  t.p = t.ts + (tok_scales ? (size_t)(k_stages + kVS) * kTile * 4 : 0);  // P parts: core matrices
  t.tab = t.p + (size_t)p_parts(tok_scales) * kOpBytes; // piece table, int32 per 16 tokens
  t.sched = t.tab + (size_t)max_pieces * 4;             // work order: pairs per tile count
                                                        // [tiles + 1], scan partials, result
  t.bar = (t.sched + (size_t)(max_pieces / 8 + 1 + kSchedExtra) * 4 + 15) / 16 * 16;
  t.misc = t.bar + (size_t)tc_barriers(k_stages) * 8;   // tmem address, abort flag, is_last
  t.rows = t.k;                                         // merge: row reference, denominator
                                                        // (after the tiles: K stage 0)
  t.total = t.misc + 16 + 1024;                         // + slack for 1024-byte alignment
  return t;
}

// ------------------------------------------------------------------ the kernel

// TS: finer-grained scales -- one dynamic scale per (token, KV head) for K and
// V (p.k_tok_scale / p.v_tok_scale, [P][Hkv][ps]), staged per tile beside the
// codes; K scales multiply the scores, V scales (divided by the head's bound
// p.v_scale[h], so that the probabilities stay in E4M3 range) the
// probabilities of the PV product, and the bound scales the output.
template <int KS, bool TS>
__global__ void __launch_bounds__(kThreads, 2) paged_decode_tc_kernel(const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const TcLayout lay = tc_layout(KS, p.split_tokens / 16, TS);
  float* sKS = reinterpret_cast<float*>(smem + lay.ts);  // [KS][128] K scales
  float* sVS = sKS + KS * kTile;                          // [kVS][128] V scales
  uint8_t* sK = smem + lay.k;
  uint8_t* sV = smem + lay.v;
  uint8_t* sP = smem + lay.p;
  int* s_tab = reinterpret_cast<int*>(smem + lay.tab);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + lay.bar);
  uint64_t* kfull_bar = bars;                  // [KS] K copies landed
  uint64_t* kempty_bar = kfull_bar + KS;       // [KS] S product of the stage's tile done
  uint64_t* kscfree_bar = kempty_bar + KS;     // [KS] TS: the softmax has read the K scales
  uint64_t* vfull_bar = kscfree_bar + KS;      // [kVS] V copies landed
  uint64_t* vempty_bar = vfull_bar + kVS;      // [kVS] PV product of the stage's tile done
  uint64_t* sfull_bar = vempty_bar + kVS;      // [2] S buffer written
  uint64_t* sfree_bar = sfull_bar + 2;         // [2] S buffer read
  uint64_t* pfull_bar = sfree_bar + 2;         // P written (and O rescaled)
  uint64_t* pvdone_bar = pfull_bar + 1;        // PV of a tile done
  uint64_t* drain_bar = pvdone_bar + 1;        // every MMA of the CTA done
  uint64_t* qready_bar = drain_bar + 1;        // Q written to tensor memory
  constexpr int PARTS = p_parts(TS);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + lay.misc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + lay.misc + 4);
  int* s_is_last = reinterpret_cast<int*>(smem + lay.misc + 8);
  float* s_rowM = reinterpret_cast<float*>(smem + lay.rows);
  float* s_rowD = s_rowM + kRows;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cid = blockIdx.x, G = gridDim.x;
  const int RB = p.row_blocks, Hs = p.Hkv * RB;
  // new rows of sequence b and its first row in q / out: uniform q_len, or
  // per sequence from the packed offsets cu_q (ragged verify, prefill chunks)
  auto qlen_of = [&](int bb) {
    return p.cu_q ? __ldg(p.cu_q + bb + 1) - __ldg(p.cu_q + bb) : p.q_len;
  };
  auto qbase_of = [&](int bb) { return p.cu_q ? __ldg(p.cu_q + bb) : bb * p.q_len; };
  auto valid_len = [&](int L, int ql) {
    return ql >= 1 && L >= ql && L <= p.max_blocks * p.ps && L <= p.max_seq_len;
  };

  // ---- invalid sequences: zero all their rows and flag them; one CTA per b
  for (int bb = cid; bb < p.B; bb += G) {
    const int L = __ldg(p.seq_lens + bb);
    const int ql = qlen_of(bb);
    if (ql == 0 || valid_len(L, ql)) continue;
    if (tid == 0) atomicOr(p.err, ATLAS_DEVERR_SEQ_LEN);
    const size_t n = (size_t)max(ql, 0) * p.Hq * kD;
    __nv_bfloat16* o = p.out + (size_t)qbase_of(bb) * p.Hq * kD;
    for (size_t idx = tid; idx < n; idx += kThreads) o[idx] = __float2bfloat16_rn(0.f);
  }

  // ---- A1, the work order: this CTA's item (sequence, segment, split),
  // longest first
  const int T = p.split_tokens;
  int b, seg, split;
  {
    int* hist = reinterpret_cast<int*>(smem + lay.sched);  // [T / 128 + 1]
    int* wsum = hist + T / kTile + 1;                       // [kWarps]
    int* res = wsum + kWarps;                               // [4]
    auto served = [&](int bb, int Lb) { return valid_len(Lb, qlen_of(bb)); };
    if (!longest_first_item<kThreads>(cid, p.B, p.seq_lens, T, Hs, served, hist, wsum, res, b,
                                      seg, split))
      return;  // past the last item (CTA-uniform)
  }

  // ---- this CTA's split (A1): tokens [t_begin, t_end) of segment (b, h, rb)
  const int sg = b * Hs + seg;
  const int h = seg / RB, rb = seg % RB;
  const int L = __ldg(p.seq_lens + b);
  const int q_len = qlen_of(b), q_base = qbase_of(b);
  if (!valid_len(L, q_len)) return;        // CTA-uniform; rows zeroed above
  const int Rtot = q_len * p.G;            // this sequence's query rows per KV head
  if (rb * kRows >= Rtot) return;          // a row block past this sequence's rows
  const int t_begin = split * T;
  if (t_begin >= L) return;
  const int t_end = min(L, t_begin + T);
  const int n_tiles = (t_end - t_begin + kTile - 1) / kTile;
  const int n_pc = (t_end - t_begin + 15) / 16;
  const int n_parts = (L + T - 1) / T;
  const bool whole = (n_parts == 1);
  const int row0 = rb * kRows;
  const int rows = min(kRows, Rtot - row0);
  // TS: the K scales are per token (applied to the scores) and p.v_scale[h] is
  // the bound of the head's per-token V scales
  const float k_scale = TS ? 1.f : __ldg(p.k_scale + h), v_scale = __ldg(p.v_scale + h);

  // ---- A0, fused append: the step's new tokens that fall in this split are
  // quantised and stored before any bulk copy reads the pages
  if (p.k_new != nullptr) {
    const int first_new = L - q_len;
    const int a0 = max(t_begin, first_new);
    const int n_new = t_end - a0;
    if (n_new > 0) {
      constexpr int CH = kD / 16;
      for (int idx = tid; idx < 2 * n_new * CH; idx += kThreads) {
        const int which = idx / (n_new * CH);  // 0 = K, 1 = V
        const int r = idx - which * n_new * CH;
        const int pos = a0 + r / CH, j = r % CH;
        const int page = __ldg(p.block_table + (size_t)b * p.max_blocks + pos / p.ps);
        if (page < 0 || page >= p.num_pages) {
          atomicOr(p.err, ATLAS_DEVERR_APPEND);
          continue;
        }
        float x[16];
        load16_as_f32(which ? p.v_new : p.k_new,
                      (((size_t)q_base + (pos - first_new)) * p.Hkv + h) * kD + 16 * j,
                      p.new_dtype, x);
        const uint4 codes = quantize16_e4m3(x, which ? v_scale : k_scale);
        const size_t head_page = (size_t)page * p.Hkv + h;
        if (!which)
          store16_k(const_cast<uint8_t*>(p.k_pages), head_page, kD, p.ps, pos % p.ps, j, codes);
        else
          store16_v(const_cast<uint8_t*>(p.v_pages), head_page, kD, p.ps, pos % p.ps, j, codes);
      }
      __threadfence();
      fence_proxy_async_global();
    }
  }

  // ---- A2, block-table gather: index of every 16-token piece of the split
  // (2048-byte blocks of the page arrays), -1 for a bad page id
  for (int k = tid; k < n_pc; k += kThreads) {
    const int t = t_begin + 16 * k;
    const int pg = t / p.ps;
    const int pid = __ldg(p.block_table + (size_t)b * p.max_blocks + pg);
    int pc = -1;
    if (pid < 0 || pid >= p.num_pages)
      atomicOr(p.err, ATLAS_DEVERR_PAGE_ID);
    else
      pc = (pid * p.Hkv + h) * (p.ps / 16) + (t - pg * p.ps) / 16;
    s_tab[k] = pc;
  }

  // softmax warps that hold at least one of the block's rows; the others
  // (and their rows of Q, S, P and O) sit the tiles out
  const int n_act = min(4, (rows + 15) / 16);
  const int my_row = 16 * (warp & 3) + (lane & 15);  // softmax warps: this thread's row
  const int my_half = lane >> 4;                     // tokens / dims 64 * half .. + 63
  float row_scale2 = 0.f;                            // score -> base-2 exponent
  int row_lim = -1;                                  // last visible key position
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      mbar_init(&kfull_bar[s], 1);
      mbar_init(&kempty_bar[s], 1);
      mbar_init(&kscfree_bar[s], 32 * n_act);
    }
    for (int s = 0; s < kVS; ++s) {
      mbar_init(&vfull_bar[s], 1);
      mbar_init(&vempty_bar[s], 1);
    }
    mbar_init(&sfull_bar[0], 1);
    mbar_init(&sfull_bar[1], 1);
    mbar_init(&sfree_bar[0], 32 * n_act);
    mbar_init(&sfree_bar[1], 32 * n_act);
    mbar_init(pfull_bar, 32 * n_act);
    mbar_init(pvdone_bar, 1);
    mbar_init(drain_bar, 1);
    mbar_init(qready_bar, 32 * n_act);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    __syncwarp();
    tmem_alloc(s_tmem, kTmemCols);
  }
  tc_fence_before();
  __syncthreads();  // table, barriers, tensor memory and appended tokens ready
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint64_t limit = ns_to_cycles(p.wait_limit_ns);  // for tc_wait and the event loops

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    // One converged warp serves two rings, K and V: a K stage is refilled as
    // soon as the S product has read it (and, with per-token scales, the
    // softmax has read its K scales), a V stage once the PV product has.
    // Each pass, lanes 0-2 test the three release barriers at once; then
    // lanes 0-7 take the K pieces of tile jk and lanes 8-15 the V pieces of
    // tile jv (either group only if its stage is free), and every lane that
    // starts a run of pieces lying back to back in the page arrays (a page of
    // 64 slots is four adjacent pieces) issues one copy for the run: a
    // tile's copies go out together, with no serial work per piece.  A
    // token-scale copy (64 bytes per piece) goes with every piece.  Bounded:
    // no progress for the wait limit raises the abort flag.
    const uint64_t policy = l2_evict_first_policy();
    const bool kg = lane < 8;
    const int gl = lane & 7;
    int jk = 0, jv = 0;
    uint64_t t_idle = sm_cycles();
    while (jk < n_tiles || jv < n_tiles) {
      bool rdy = false;
      if (lane == 0)
        rdy = jk < n_tiles &&
              (jk < KS || mbar_test(&kempty_bar[jk % KS], (uint32_t)(((jk / KS) - 1) & 1)));
      else if (lane == 1)
        rdy = !TS || jk >= n_tiles || jk < KS ||
              mbar_test(&kscfree_bar[jk % KS], (uint32_t)(((jk / KS) - 1) & 1));
      else if (lane == 2)
        rdy = jv < n_tiles &&
              (jv < kVS || mbar_test(&vempty_bar[jv % kVS], (uint32_t)(((jv / kVS) - 1) & 1)));
      const unsigned r = __ballot_sync(kFull, rdy);
      const bool do_k = (r & 3u) == 3u, do_v = (r & 4u) != 0;
      if (!do_k && !do_v) {
        bool stop = false;
        if (lane == 0) {
          if (*s_abort) {
            stop = true;
          } else if (sm_cycles() - t_idle > limit) {
            *s_abort = 1;
            stop = true;
          }
        }
        if (__shfl_sync(kFull, stop ? 1 : 0, 0)) break;
        __nanosleep(32);
        continue;
      }
      if (lane == 0) t_idle = sm_cycles();
      const int j = kg ? jk : jv;
      const bool mine = lane < 16 && (kg ? do_k : do_v) &&
                        !(p.test_skip_unit == j && cid == 0);  // lost copy (tests only)
      const int st = kg ? j % KS : j % kVS;
      uint64_t* fb = kg ? &kfull_bar[st] : &vfull_bar[st];
      const int k = 8 * j + gl;
      const int piece = (mine && k < n_pc) ? s_tab[k] : -1;
      // a run starts at a valid piece whose left neighbour (same group) is
      // not the piece before it in the page arrays
      const int left = __shfl_up_sync(kFull, piece, 1);
      const bool adj = gl > 0 && piece >= 0 && left >= 0 && left + 1 == piece;
      const unsigned adj_mask = __ballot_sync(kFull, adj);
      const unsigned valid_mask = __ballot_sync(kFull, piece >= 0);
      const bool starts = piece >= 0 && !adj;
      // run length: this piece plus the adjacent pieces right after it
      const int run = starts ? __ffs(~(adj_mask >> (lane + 1))) : 0;
      const unsigned grp_valid = valid_mask & (kg ? 0x000000FFu : 0x0000FF00u);
      if (mine && gl == 0) {
        const uint32_t bytes = (uint32_t)__popc(grp_valid) * (kPiece + (TS ? 64 : 0));
        if (bytes == 0)
          mbar_arrive(fb);
        else
          mbar_arrive_expect_tx(fb, bytes);
      }
      __syncwarp();
      if (starts) {
        bulk_load((kg ? sK : sV) + (size_t)st * kTileBytes + gl * kPiece,
                  (kg ? p.k_pages : p.v_pages) + (size_t)piece * kPiece, (uint32_t)run * kPiece,
                  fb, policy);
        if constexpr (TS) {  // the run's K or V scales (64 bytes per piece)
          bulk_load((kg ? sKS : sVS) + (size_t)st * kTile + 16 * gl,
                    (kg ? p.k_tok_scale : p.v_tok_scale) + (size_t)piece * 16,
                    (uint32_t)run * 64, fb, policy);
        }
      }
      if (do_k) ++jk;
      if (do_v) ++jv;
    }
    if (*s_abort && lane == 0) {
      // drain: copies of the last stages issued may still be in flight
      for (int j = max(0, jk - KS); j < jk; ++j)
        mbar_wait_bounded(&kfull_bar[j % KS], (uint32_t)((j / KS) & 1), p.wait_limit_ns);
      for (int j = max(0, jv - kVS); j < jv; ++j)
        mbar_wait_bounded(&vfull_bar[j % kVS], (uint32_t)((j / kVS) & 1), p.wait_limit_ns);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f8(64, 64);
      // operand descriptors of the first tile, stage 0; every other operand
      // is one of these plus a byte offset / 16 in the start-address field
      // (all addresses stay below 256 KB, so the field never carries)
      const uint64_t dp = smem_desc(smem_u32(sP), 128, 1024, 0);
      const uint64_t dk = smem_desc(smem_u32(sK), 16, 1024, 2);
      const uint64_t dv = smem_desc(smem_u32(sV), kPiece, 128, 0);
      bool ok = tc_wait(qready_bar, 0, s_abort, limit);
      auto issue_pv = [&](int k) {  // O += P . V for tile k
        const int st = k % kVS;
        const int tok = t_end - (t_begin + kTile * k);  // valid tokens of the tile (>= 1)
        const int nks = min(4, (tok + 31) / 32);       // 32-token k-steps holding any
        const uint64_t dvs = dv + (uint64_t)((st * kTileBytes) >> 4);
#pragma unroll
        for (int dh = 0; dh < 2; ++dh) {
          const uint32_t d = tmem + ((uint32_t)(16 * dh) << 16) + kColO;
#pragma unroll
          for (int part = 0; part < PARTS; ++part)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              if (ks >= nks) break;
              mma_f8(d, dp + (uint64_t)((part * kOpBytes + ks * 256) >> 4),
                     dvs + (uint64_t)((ks * 2 * kPiece + dh * 1024) >> 4), idesc,
                     (k > 0 || part > 0 || ks > 0) ? 1u : 0u);
            }
        }
        mma_commit(&vempty_bar[st]);
        mma_commit(pvdone_bar);
      };
      auto issue_s = [&](int j) {  // S = (Qhi + Qlo) . K^T for tile j
        const int st = j % KS, sb = j & 1;
        const uint64_t dks = dk + (uint64_t)((st * kTileBytes) >> 4);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (t_begin + kTile * j + 64 * half >= t_end) break;  // no token in this half
          // Q rows sit in the same lanes as the S rows they produce
          const uint32_t lanes = (uint32_t)(16 * half) << 16;
#pragma unroll
          for (int part = 0; part < 2; ++part)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_f8_ta(tmem + lanes + kColS + 64 * sb, tmem + lanes + kColQ + 32 * part + 8 * ks,
                        dks + (uint64_t)((half * 8192 + ks * 32) >> 4), idesc,
                        (part > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&kempty_bar[st]);
        mma_commit(&sfull_bar[sb]);
      };
      // Event loop: S(js) once the K of tile js has landed and its S buffer
      // is free (at most two S tiles ahead of the PV products), PV(jp) once
      // the softmax has written P(jp) and the V of tile jp has landed --
      // whichever is ready first, so that a PV never waits behind the next
      // tile's copies.  Bounded: no progress for the wait limit raises the
      // abort flag.
      int js = 0, jp = 0;
      uint64_t t_idle = sm_cycles();
      while (ok && jp < n_tiles) {
        bool progressed = false;
        if (js < n_tiles && js < jp + 2 &&
            mbar_test(&kfull_bar[js % KS], (uint32_t)((js / KS) & 1)) &&
            (js < 2 || mbar_test(&sfree_bar[js & 1], (uint32_t)(((js >> 1) - 1) & 1)))) {
          tc_fence_after();
          issue_s(js);
          ++js;
          progressed = true;
        }
        if (jp < js && mbar_test(pfull_bar, (uint32_t)(jp & 1)) &&
            mbar_test(&vfull_bar[jp % kVS], (uint32_t)((jp / kVS) & 1))) {
          tc_fence_after();
          issue_pv(jp);
          ++jp;
          progressed = true;
        }
        if (progressed) {
          t_idle = sm_cycles();
        } else if (*s_abort) {
          ok = false;
        } else if (sm_cycles() - t_idle > limit) {
          *s_abort = 1;
          ok = false;
        } else {
          __nanosleep(32);  // leave issue slots to the softmax warp of this SM quarter
        }
      }
      // every MMA issued so far has completed before tensor memory is released
      mma_commit(drain_bar);
      mbar_wait_bounded(drain_bar, 0, p.wait_limit_ns);
    }
  } else if (warp < n_act) {
    // ------------------------------------------------------------ softmax
    // (first the Q rows, while the producer's first copies are in flight)
  // ---- Q rows as E4M3 hi + lo with a per-row power-of-two scale, written
  // to tensor memory as the A operand of the S product: row r in the lanes
  // of the S rows it produces -- both lane r % 16 and lane 16 + r % 16 of
  // warp r / 16's quadrant, for the two token halves -- dims 4c .. 4c + 3 of
  // a part in column c (hi: kColQ + c, lo: kColQ + 32 + c)
  {
    const int r = my_row, rr = row0 + r;
    float x[64];
    if (r < rows) {
      const int i = rr / p.G, hq = h * p.G + rr % p.G;
      const uint4* src = reinterpret_cast<const uint4*>(
          p.q + (((size_t)q_base + i) * p.Hq + hq) * kD + 64 * my_half);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 w = __ldg(src + c);
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          x[8 * c + 2 * k] = __uint_as_float(wv[k] << 16);
          x[8 * c + 2 * k + 1] = __uint_as_float(wv[k] & 0xFFFF0000u);
        }
      }
      row_lim = L - q_len + i;
    } else {
#pragma unroll
      for (int k = 0; k < 64; ++k) x[k] = 0.f;
    }
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < 64; ++k) amax = fmaxf(amax, fabsf(x[k]));
    amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 16));
    // a = 2^(135 - e) puts amax in [256, 512); halve it if amax * a > 448
    float a = 1.f;
    if (amax > 0.f) {
      const int e = (int)((__float_as_uint(amax) >> 23) & 0xFF);
      a = __uint_as_float((uint32_t)min(254, max(1, 262 - e)) << 23);
      if (amax * a > 448.f) a *= 0.5f;
    }
    row_scale2 = k_scale * p.qk_scale_log2 / a;
    uint32_t hw[16], lw[16];  // this thread's 64 dims: word 4 cc + w4 = dims 16 cc + 4 w4 ..
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
#pragma unroll
      for (int w4 = 0; w4 < 4; ++w4) {
        const int k0 = 16 * cc + 4 * w4;
        const float y0 = x[k0] * a, y1 = x[k0 + 1] * a, y2 = x[k0 + 2] * a, y3 = x[k0 + 3] * a;
        const uint32_t h01 = f32x2_to_e4m3x2(y0, y1), h23 = f32x2_to_e4m3x2(y2, y3);
        const uint32_t f01 = e4m3x2_to_f16x2(h01), f23 = e4m3x2_to_f16x2(h23);
        const float2 b01 = __half22float2(*reinterpret_cast<const __half2*>(&f01));
        const float2 b23 = __half22float2(*reinterpret_cast<const __half2*>(&f23));
        const uint32_t l01 = f32x2_to_e4m3x2(y0 - b01.x, y1 - b01.y);
        const uint32_t l23 = f32x2_to_e4m3x2(y2 - b23.x, y3 - b23.y);
        hw[4 * cc + w4] = h01 | (h23 << 16);
        lw[4 * cc + w4] = l01 | (l23 << 16);
      }
    }
    // the whole row in this thread's lane: the partner (lane ^ 16) holds the
    // other 64 dims
    const uint32_t qa = tmem + ((uint32_t)(32 * warp) << 16) + kColQ;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      uint32_t row[32];
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint32_t own = part ? lw[c] : hw[c];
        const uint32_t other = __shfl_xor_sync(kFull, own, 16);
        row[c] = my_half ? other : own;
        row[16 + c] = my_half ? own : other;
      }
      tmem_st32(qa + 32 * part, row);
    }
    tc_fence_before();
    mbar_arrive(qready_bar);
  }

    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    const bool row_ok = my_row < rows;
    float m_run = -INFINITY, l_run = 0.f;
    bool aborted = false;
    for (int j = 0; j < n_tiles; ++j) {
      const int sb = j & 1, sk = j % KS, sv_st = j % kVS;
      const uint32_t vpar = (uint32_t)((j / kVS) & 1);
      bool ok = tc_wait(&sfull_bar[sb], (uint32_t)((j >> 1) & 1), s_abort, limit);
      if (!__all_sync(kFull, ok)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      uint32_t sv[64];
      {
        uint32_t a[32], c[32];
        tmem_ld32(tmem + lane_base + kColS + 64 * sb, a);
        tmem_ld32(tmem + lane_base + kColS + 64 * sb + 32, c);
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          sv[k] = a[k];
          sv[32 + k] = c[k];
        }
      }
      tc_fence_before();
      mbar_arrive(&sfree_bar[sb]);

      // mask (A5): tokens past the split, in a bad page, or after the row's
      // limit (a row past the block's rows has limit -1: all masked)
      const int t0 = t_begin + kTile * j + 64 * my_half;
      const int lim = min(t_end - 1, row_lim);
      float x[64];
      bool pc_ok[4];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) pc_ok[q4] = s_tab[(t0 - t_begin) / 16 + q4] >= 0;
      const bool clean = (t0 + 63 <= lim) && pc_ok[0] && pc_ok[1] && pc_ok[2] && pc_ok[3];
      if constexpr (TS) {  // per-token K scales
        const float4* ksc = reinterpret_cast<const float4*>(sKS + (size_t)sk * kTile +
                                                             64 * my_half);
#pragma unroll
        for (int k4 = 0; k4 < 16; ++k4) {
          const float4 f = ksc[k4];
          sv[4 * k4] = __float_as_uint(__uint_as_float(sv[4 * k4]) * f.x);
          sv[4 * k4 + 1] = __float_as_uint(__uint_as_float(sv[4 * k4 + 1]) * f.y);
          sv[4 * k4 + 2] = __float_as_uint(__uint_as_float(sv[4 * k4 + 2]) * f.z);
          sv[4 * k4 + 3] = __float_as_uint(__uint_as_float(sv[4 * k4 + 3]) * f.w);
        }
        mbar_arrive(&kscfree_bar[sk]);  // the K producer may refill the stage
      }
      if (clean) {
#pragma unroll
        for (int k = 0; k < 64; ++k) x[k] = __uint_as_float(sv[k]) * row_scale2;
      } else {
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          const bool ok_t = t0 + k <= lim && pc_ok[k >> 4];
          x[k] = ok_t ? __uint_as_float(sv[k]) * row_scale2 : -INFINITY;
        }
      }

      // online softmax (A6): the row's reference moves only when a score
      // exceeds it by more than 0.5; both threads of the row decide alike
      float mx;
      {  // eight independent chains, then a tree
        float m8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) m8[e] = x[e];
#pragma unroll
        for (int k = 8; k < 64; ++k) m8[k & 7] = fmaxf(m8[k & 7], x[k]);
        mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      }
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
      const bool move = mx > m_run + 0.5f;
      float alpha = 1.f;
      if (move) {
        alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - mx);
        m_run = mx;
        l_run *= alpha;
      }
      // O (rescaled when a row's reference moved) and P's buffer are free
      // once the previous tile's PV is done: the exponentials and the E4M3
      // parts below run while it is in flight, and the wait comes after them
      // p = 2^(x - m + 8) -> E4M3 parts, in V's slot order inside each
      // 16-token chunk (word c = slots 2c, 2c+1, 2c+8, 2c+9)
      const float off = 8.f - ((m_run == -INFINITY) ? 0.f : m_run);
      float pr[64];
      float ls8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < 64; ++k) {
        pr[k] = fast_exp2(x[k] + off);
        ls8[k & 7] += pr[k];
      }
      l_run += ((ls8[0] + ls8[1]) + (ls8[2] + ls8[3])) + ((ls8[4] + ls8[5]) + (ls8[6] + ls8[7]));
      if constexpr (TS) {  // p * v_scale[t] / bound: at most p (masked tokens stay 0)
        ok = tc_wait(&vfull_bar[sv_st], vpar, s_abort, limit);  // V scales
        if (!__all_sync(kFull, ok)) {
          aborted = true;
          break;
        }
        const float inv_bound = 1.f / v_scale;
        const float4* vsc = reinterpret_cast<const float4*>(sVS + (size_t)sv_st * kTile +
                                                             64 * my_half);
#pragma unroll
        for (int k4 = 0; k4 < 16; ++k4) {
          const float4 f = vsc[k4];
          const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k = 4 * k4 + e;
            pr[k] = pr[k] > 0.f ? pr[k] * (fv[e] * inv_bound) : 0.f;
          }
        }
      }
      uint32_t pw[PARTS][4][4];  // [part][16-token chunk][word]
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t a0[PARTS], a1[PARTS];
          split_pair<PARTS>(pr[16 * cc + 2 * c4], pr[16 * cc + 2 * c4 + 1], a0);
          split_pair<PARTS>(pr[16 * cc + 2 * c4 + 8], pr[16 * cc + 2 * c4 + 9], a1);
#pragma unroll
          for (int q = 0; q < PARTS; ++q) pw[q][cc][c4] = a0[q] | (a1[q] << 16);
        }
      if (j > 0) {
        ok = tc_wait(pvdone_bar, (uint32_t)((j - 1) & 1), s_abort, limit);
        if (!__all_sync(kFull, ok)) {
          aborted = true;
          break;
        }
        if (__any_sync(kFull, move)) {  // rescale the moved rows' O (A7)
          tc_fence_after();
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            uint32_t o[32];
            const uint32_t ta = tmem + lane_base + kColO + 32 * c2;
            tmem_ld32(ta, o);
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st32(ta, o);
          }
        }
      }
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int offp = (my_row >> 3) * 1024 + (4 * my_half + cc) * 128 + (my_row & 7) * 16;
#pragma unroll
        for (int q = 0; q < PARTS; ++q)
          *reinterpret_cast<uint4*>(sP + q * kOpBytes + offp) =
              make_uint4(pw[q][cc][0], pw[q][cc][1], pw[q][cc][2], pw[q][cc][3]);
      }
      // V slots that hold no valid token of this tile (past the split, bad
      // page) are zeroed, so that 0 * garbage never reaches O
      const int tile0 = t_begin + kTile * j;
      bool dirty = tile0 + kTile > t_end;
#pragma unroll
      for (int pc = 0; pc < 8; ++pc) {
        const int k = 8 * j + pc;
        dirty |= (k < n_pc && s_tab[k] < 0);
      }
      if (dirty) {
        ok = tc_wait(&vfull_bar[sv_st], vpar, s_abort, limit);
        if (!__all_sync(kFull, ok)) {
          aborted = true;
          break;
        }
        for (int d = tid; d < kD; d += 32 * n_act) {  // one V row of every piece
          for (int pc = 0; pc < 8; ++pc) {
            const int k = 8 * j + pc;
            const int nvalid =
                (k < n_pc && s_tab[k] >= 0) ? min(16, t_end - (tile0 + 16 * pc)) : 0;
            if (nvalid >= 16) continue;
            uint8_t* vrow = sV + (size_t)sv_st * kTileBytes + pc * kPiece + d * 16;
            if (nvalid <= 0) {
              *reinterpret_cast<uint4*>(vrow) = make_uint4(0u, 0u, 0u, 0u);
            } else {
              for (int t = nvalid; t < 16; ++t) vrow[group_pos(t)] = 0;
            }
          }
        }
      }
      fence_proxy_async_shared();
      tc_fence_before();
      mbar_arrive(pfull_bar);
    }

    // ---- epilogue: O / l of this split -> output rows or the split's partial
    if (!aborted) {
      bool ok = tc_wait(pvdone_bar, (uint32_t)((n_tiles - 1) & 1), s_abort, limit);
      if (!__all_sync(kFull, ok)) aborted = true;
    }
    if (!aborted) {
      tc_fence_after();
      uint32_t o[64];
      {
        uint32_t a[32], c[32];
        tmem_ld32(tmem + lane_base + kColO, a);
        tmem_ld32(tmem + lane_base + kColO + 32, c);
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          o[k] = a[k];
          o[32 + k] = c[k];
        }
      }
      const float den = l_run + __shfl_xor_sync(kFull, l_run, 16);
      if (row_ok) {
        const int rr = row0 + my_row;
        const int i = rr / p.G, hq = h * p.G + rr % p.G;
        if (whole) {
          const float inv = den > 0.f ? v_scale / den : 0.f;
          uint4* dst = reinterpret_cast<uint4*>(
              p.out + (((size_t)q_base + i) * p.Hq + hq) * kD + 64 * my_half);
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const __nv_bfloat162 v2 =
                  __floats2bfloat162_rn(__uint_as_float(o[8 * c8 + 2 * k]) * inv,
                                        __uint_as_float(o[8 * c8 + 2 * k + 1]) * inv);
              w[k] = *reinterpret_cast<const uint32_t*>(&v2);
            }
            dst[c8] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          const float inv = den > 0.f ? 1.f / den : 0.f;
          const size_t slot = (size_t)sg * p.num_splits + split;
          float4* dst = reinterpret_cast<float4*>(p.part_o + (slot * kRows + my_row) * kD +
                                                  64 * my_half);
#pragma unroll
          for (int c4 = 0; c4 < 16; ++c4)
            dst[c4] = make_float4(__uint_as_float(o[4 * c4]) * inv,
                                  __uint_as_float(o[4 * c4 + 1]) * inv,
                                  __uint_as_float(o[4 * c4 + 2]) * inv,
                                  __uint_as_float(o[4 * c4 + 3]) * inv);
          // the log2-sum-exp carries the 2^8 of p; it cancels in the merge
          if (my_half == 0)
            p.part_lse[slot * kRows + my_row] = den > 0.f ? m_run + __log2f(den) : -INFINITY;
        }
      }
    }
  }

  // ---- teardown: every tcgen05 operation is complete (drained above)
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (*s_abort) {
    if (tid == 0) atomicOr(p.err, ATLAS_DEVERR_TIMEOUT);
    return;
  }
  if (whole) return;

  // ---- A8 -> A9: the CTA that finishes the segment last merges its splits
  __threadfence();
  __syncthreads();
  if (tid == 0) *s_is_last = (atomicAdd(p.counters + sg, 1) == n_parts - 1);
  __syncthreads();
  if (!*s_is_last) return;
  __threadfence();
  const size_t s0 = (size_t)sg * p.num_splits;
  for (int r = tid; r < rows; r += kThreads) {
    float M = -INFINITY, den = 0.f;
    for (int sl = 0; sl < n_parts; ++sl) {
      const float v = __ldcg(p.part_lse + (s0 + sl) * kRows + r);
      if (v == -INFINITY) continue;
      if (v > M) {
        den = den * fast_exp2(M - v) + 1.f;
        M = v;
      } else {
        den += fast_exp2(v - M);
      }
    }
    s_rowM[r] = M;
    s_rowD[r] = den;
  }
  __syncthreads();
  constexpr int C4 = kD / 4;
  for (int idx = tid; idx < rows * C4; idx += kThreads) {
    const int r = idx / C4, d0 = 4 * (idx - r * C4);
    const float M = s_rowM[r], den = s_rowD[r];
    float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (den > 0.f) {
#pragma unroll 4
      for (int sl = 0; sl < n_parts; ++sl) {
        const float wgt = fast_exp2(__ldcg(p.part_lse + (s0 + sl) * kRows + r) - M);
        const float4 v =
            __ldcg(reinterpret_cast<const float4*>(p.part_o + ((s0 + sl) * kRows + r) * kD + d0));
        o4.x += wgt * v.x; o4.y += wgt * v.y; o4.z += wgt * v.z; o4.w += wgt * v.w;
      }
    }
    const float inv = den > 0.f ? v_scale / den : 0.f;
    const int rr = row0 + r;
    const int i = rr / p.G, hq = h * p.G + rr % p.G;
    __nv_bfloat16* dst = p.out + (((size_t)q_base + i) * p.Hq + hq) * kD + d0;
    const __nv_bfloat162 lo = __floats2bfloat162_rn(o4.x * inv, o4.y * inv);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(o4.z * inv, o4.w * inv);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&lo);
    pk.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(dst) = pk;
  }
  if (tid == 0) p.counters[sg] = 0;  // ready for the next call on this stream
}

}  // namespace

size_t decode_tc_smem_bytes(int stages, int split_tokens, bool tok_scales) {
  return tc_layout(stages, split_tokens / 16, tok_scales).total;
}

cudaError_t launch_decode_tc(const DecodeParams& p, int stages, long long grid,
                             cudaStream_t stream) {
  if (grid < 1 || grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  if (p.D != kD || p.split_tokens % kTile != 0) return cudaErrorInvalidValue;
  // at least 80 KB of shared memory per CTA: never more than two CTAs per SM,
  // so the two 256-column tensor-memory allocations always fit (an
  // allocation that cannot be served would wait)
  const bool ts = p.k_tok_scale != nullptr;
  size_t smem = decode_tc_smem_bytes(stages, p.split_tokens, ts);
  if (smem < 80 * 1024) smem = 80 * 1024;
  auto go = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
  };
  if (stages == 2) return ts ? go(paged_decode_tc_kernel<2, true>) : go(paged_decode_tc_kernel<2, false>);
  if (stages == 3) return ts ? go(paged_decode_tc_kernel<3, true>) : go(paged_decode_tc_kernel<3, false>);
  return cudaErrorInvalidValue;
}

}  // namespace atlas
