// Internal declarations shared by the kernels and the C-ABI layer.
// Device helpers here wrap single PTX instructions (conversion,
// register-matrix transpose, base-2 exponential, mbarriers, bulk copies); none
// re-implements a math-library routine.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "atlas_kv.h"

namespace atlas {

// ---------------------------------------------------------------- parameters

struct AppendParams {
  const void* k_new;          // [B][n_new][Hkv][D] f32 or bf16
  const void* v_new;
  int dtype;                  // ATLAS_DTYPE_*
  uint8_t* k_pages;           // [P][Hkv][ps][D]  (token-major)
  uint8_t* v_pages;           // [P][Hkv][ps/16][D][16]  (16-slot groups, head-dim-major)
  const float* k_scale;       // [Hkv]
  const float* v_scale;
  const int32_t* block_table; // [B][max_blocks]
  const int32_t* start_pos;   // [B]
  int32_t* err;               // device error word
  int batch, n_new, Hkv, D, ps, num_pages, max_blocks;
  // finer-grained scales (nullptr: the per-head k_scale / v_scale): one
  // dynamic scale per (token, KV head), [P][Hkv][ps], and the per-head bound
  // of the V scales, [Hkv] (raised with atomicMax)
  float* k_tok_scale;
  float* v_tok_scale;
  float* v_scale_bound;
};

struct DecodeParams {
  const __nv_bfloat16* q;     // [B][q_len][Hq][D]
  const uint8_t* k_pages;     // [P][Hkv][ps][D]  (token-major)
  const uint8_t* v_pages;     // [P][Hkv][ps/16][D][16]  (16-slot groups, head-dim-major)
  const float* k_scale;       // [Hkv]
  const float* v_scale;
  const int32_t* block_table; // [B][max_blocks]
  const int32_t* seq_lens;    // [B]
  const int32_t* cu_q;        // nullptr: q_len rows per sequence; else [B + 1] packed row
                              // offsets (q, out are [cu_q[B]][Hq][D], q_len = the largest)
  __nv_bfloat16* out;         // [B][q_len][Hq][D]
  float* part_o;              // [slots][rows_per_cta][D]  (partials of cut segments)
  float* part_lse;            // [slots][rows_per_cta]     (log2-domain LSE)
  int32_t* counters;          // [B][Hkv][row_blocks], zero between calls
  int32_t* err;               // device error word
  int B, Hq, Hkv, G, q_len, D, ps, num_pages, max_blocks, max_seq_len;
  int row_blocks;
  int max_units;              // most 32-token units one CTA is given
  int max_portions;           // most segments one CTA's range meets
  int grid_mode;              // 1: grid partition (CTA = split of a segment), 0: balanced
  int num_splits, split_tokens;  // grid partition
  float qk_scale_log2;        // sm_scale * log2(e); k_scale[h] is folded in per head
  // fused append (A0): when k_new != nullptr the kernel first quantises and
  // writes the q_len new tokens of each sequence, positions L - q_len .. L - 1
  const void* k_new;          // [B][q_len][Hkv][D] f32 or bf16, or nullptr
  const void* v_new;
  int new_dtype;              // ATLAS_DTYPE_*
  // bounded waits: wall-clock limit of every mbarrier wait (ns)
  unsigned long long wait_limit_ns;
  // test-only lost-copy injection: when >= 0, CTA 0's first K/V stream never
  // issues the bulk copies of its unit number test_skip_unit, so the wait for
  // them runs out (no copy is in flight for that stage); -1 in normal use
  int test_skip_unit;
  // finer-grained scales (tensor-core kernel only): per-(token, KV head) K and
  // V scales [P][Hkv][ps]; then v_scale holds the heads' bounds of the V scales
  // and k_scale is not read.  nullptr: the per-head scales.
  const float* k_tok_scale;
  const float* v_tok_scale;
};

constexpr unsigned long long kDefaultWaitLimitNs = 200ull * 1000 * 1000;

cudaError_t launch_fp8_append(const AppendParams& p, int num_sms, cudaStream_t stream);

struct RopeAppendParams {
  const __nv_bfloat16* qkv;   // [B][n_new][Hq + 2 Hkv][D]: query, key, value heads
  const float* cos_sin;       // [max_pos][D]: cos in columns 0..D/2-1, sin in D/2..D-1
  int max_pos;
  __nv_bfloat16* q_out;       // [B][n_new][Hq][D]: rotated queries
  uint8_t* k_pages;
  uint8_t* v_pages;
  const float* k_scale;       // [Hkv]
  const float* v_scale;
  const int32_t* block_table; // [B][max_blocks]
  const int32_t* start_pos;   // [B]
  int32_t* err;
  int batch, n_new, Hq, Hkv, D, ps, num_pages, max_blocks;
};

cudaError_t launch_rope_append(const RopeAppendParams& p, cudaStream_t stream);

// Greedy MTP acceptance: one CTA per logits row; counters: int32 [batch],
// zero before the launch and left zero.
cudaError_t launch_mtp_accept(const void* logits, int dtype, int batch, int num_drafts, int vocab,
                              const int32_t* drafts, int32_t* targets, int32_t* n_accepted,
                              int32_t* next_token, int32_t* counters, cudaStream_t stream);

// Launch shape of the decode kernel for one call (A1).  A segment is
// (sequence, KV head, row group of rows_per_cta query rows); a unit is 32 KV
// tokens of a segment.
//  * Grid partition: CTA = one split of split_tokens tokens of one segment
//    (num_splits per segment, as if every sequence were max_seq_len long;
//    splits past a sequence's end exit at once).  The hardware hands CTAs to
//    SMs as they free up, which evens out SMs that get slower memory service.
//  * Balanced partition: the units of all segments, in (b, h, rg) order, are
//    cut into `grid` equal ranges, one per CTA, whatever the length mix.
// Either way a segment cut in several parts leaves one partial per part,
// merged by log-sum-exp by the CTA that finishes the segment last.
enum { kPartitionAuto = 0, kPartitionGrid = 1, kPartitionBalanced = 2 };

struct DecodeLaunch {
  int rows_per_warp, rbg, rows_per_cta, row_blocks, stages;
  int waves;             // automatic grid: this many CTAs per resident CTA slot
  int grid_mode;         // 1: grid partition, 0: balanced
  int split_tokens;      // grid partition: tokens per split (a multiple of 64)
  int num_splits;        // grid partition: splits per segment
  long long segs;        // B * Hkv * row_blocks
  long long units_max;   // segs * ceil(max_seq_len / 32): units if every L were max_seq_len
  long long grid;        // CTAs
  int max_units;         // units of the largest range
  int max_portions;      // segments the largest range can meet
  long long slots;       // partial slots (0: no segment is ever cut)
};

constexpr int kMaxUnitsPerCta = 1024;  // bounds the per-CTA unit table in shared memory

// Which decode kernel serves a call: the FP8 warp-MMA kernel (mma.sync, any
// row count, head_dim 64 or 128) or the 5th-generation tensor-core kernel
// (tcgen05.mma with accumulators in tensor memory, head_dim 128, blocks of 64
// query rows).  Automatic: tcgen05 when head_dim is 128 and a KV head has at
// least kTcMinRows query rows (q_len * G), where QK^T and PV are real
// contractions; the warp-MMA kernel otherwise.
enum { kKernelAuto = 0, kKernelWarpMma = 1, kKernelTc = 2 };
constexpr int kTcMinRows = 16;

inline bool use_tc_kernel(int kernel, int head_dim, int q_len, int G) {
  if (kernel == kKernelWarpMma) return false;
  if (kernel == kKernelTc) return true;
  return head_dim == 128 && q_len * G >= kTcMinRows;
}

// Launch plan of the tensor-core kernel: grid partition (CTA = one split of a
// (sequence, KV head, 64-row block) segment, splits of a multiple of 128
// tokens), two resident CTAs per SM.  split_tokens > 0 overrides the split
// length (rounded up to a multiple of 128).
inline DecodeLaunch plan_decode_tc(int B, int Hq, int Hkv, int q_len, int max_seq_len, int sms,
                                   int split_tokens, int stages_override, int waves = 1) {
  DecodeLaunch L;
  L.waves = waves < 1 ? 1 : waves;
  const int R = q_len * (Hq / Hkv);
  L.rows_per_warp = 16;
  L.rbg = 4;
  L.rows_per_cta = 64;
  L.row_blocks = (R + 63) / 64;
  L.stages = stages_override > 0 ? stages_override : 3;  // K ring depth (the V ring has 2)
  L.segs = (long long)B * Hkv * L.row_blocks;
  L.units_max = L.segs * (((long long)max_seq_len + 31) / 32);
  L.grid_mode = 1;
  const long long resident = (long long)sms * 2;
  long long T;
  if (split_tokens > 0) {
    T = (split_tokens + 127) / 128 * 128;
  } else {
    // as the warp-MMA grid partition: splits for two to four waves of
    // resident CTAs if every sequence were max_seq_len long, but not under
    // 2048 tokens unless one wave needs shorter ones; multiple of 128 in
    // [256, 8192]
    const long long segs = L.segs > 0 ? L.segs : 1;
    auto split_for = [&](long long ctas) {
      long long want = (ctas + segs - 1) / segs;
      if (want < 1) want = 1;
      const long long t = ((long long)max_seq_len + want - 1) / want;
      return (t + 127) / 128 * 128;
    };
    const long long one_wave = split_for(resident * L.waves);
    const long long two_waves = split_for(2 * resident * L.waves);
    T = 128;
    while (2 * T <= two_waves) T *= 2;
    const long long lo = one_wave < 2048 ? one_wave : 2048;
    if (T < lo) T = lo;
    if (T < 256) T = 256;
    if (T > 8192) T = 8192;
  }
  L.split_tokens = (int)T;
  L.num_splits = (int)(((long long)max_seq_len + T - 1) / T);
  if (L.num_splits < 1) L.num_splits = 1;
  L.grid = L.segs * L.num_splits;
  L.max_units = (int)((T + 31) / 32);
  L.max_portions = 1;
  L.slots = L.num_splits > 1 ? L.segs * L.num_splits : 0;
  return L;
}

// Resident CTAs per SM the kernel is built for (its __launch_bounds__).
inline int decode_target_occupancy(int rows_per_warp, int rbg) {
  return (rows_per_warp <= 8 && rbg == 1) ? 3 : 2;
}

// split_tokens > 0: splits / ranges of about split_tokens KV tokens; 0: the
// automatic choice.  partition: kPartition*.  Automatic: the balanced
// partition when one K/V stream serves the whole CTA (rbg 4: no in-CTA
// combine, so range portions switch cheaply, and ragged lengths balance),
// the grid partition otherwise.
// rows_per_cta: 0 = automatic (the smallest of 4, 8, 16, 32, 64 that holds
// all q_len * G rows of a KV head), else one of those (more row blocks).
inline DecodeLaunch plan_decode(int B, int Hq, int Hkv, int q_len, int max_seq_len, int sms,
                                int split_tokens, int stages_override, int partition,
                                int waves = 1, int rows_per_cta = 0) {
  DecodeLaunch L;
  L.waves = waves < 1 ? 1 : waves;
  const int G = Hq / Hkv;
  const int R = q_len * G;
  const int rc = rows_per_cta > 0 ? rows_per_cta : (R <= 4 ? 4 : R <= 8 ? 8 : R <= 16 ? 16 : R <= 32 ? 32 : 64);
  L.rows_per_warp = rc <= 8 ? rc : 16;  // 4: hi | lo packed MMA columns
  L.rbg = rc <= 16 ? 1 : rc / 16;        // warps sharing one K/V stream
  L.rows_per_cta = L.rows_per_warp * L.rbg;
  L.row_blocks = (R + L.rows_per_cta - 1) / L.rows_per_cta;
  L.stages = stages_override > 0 ? stages_override : (L.rbg == 1 ? 2 : 3);
  L.segs = (long long)B * Hkv * L.row_blocks;
  const long long seg_units = ((long long)max_seq_len + 31) / 32;
  L.units_max = L.segs * seg_units;
  const long long resident = (long long)sms * decode_target_occupancy(L.rows_per_warp, L.rbg);
  L.grid_mode = (partition == kPartitionGrid || (partition == kPartitionAuto && L.rbg != 4));
  if (L.grid_mode) {
    long long T;
    if (split_tokens > 0) {
      T = (split_tokens + 63) / 64 * 64;
    } else {
      // splits for at least two waves of resident CTAs if every sequence were
      // max_seq_len long (the split for two waves rounded down to a power of
      // two: two to four waves), so that the hardware can even out the SMs;
      // but a split under 2048 tokens spends too much of its time in the
      // prologue -- unless even one wave needs shorter splits.  Multiple of
      // 64 in [256, 8192].  (Measured on the long-context workload: 4096-token
      // splits 148 µs, 4736: 160 µs, 3072: 167 µs; LLaMA-shaped: 2048 best.)
      const long long segs = L.segs > 0 ? L.segs : 1;
      auto split_for = [&](long long ctas) {
        long long want = (ctas + segs - 1) / segs;
        if (want < 1) want = 1;
        const long long t = ((long long)max_seq_len + want - 1) / want;
        return (t + 63) / 64 * 64;
      };
      const long long one_wave = split_for(resident * L.waves);
      const long long two_waves = split_for(2 * resident * L.waves);
      T = 64;
      while (2 * T <= two_waves) T *= 2;
      const long long lo = one_wave < 2048 ? one_wave : 2048;
      if (T < lo) T = lo;
      if (T < 256) T = 256;
      if (T > 8192) T = 8192;
    }
    L.split_tokens = (int)T;
    L.num_splits = (int)(((long long)max_seq_len + T - 1) / T);
    if (L.num_splits < 1) L.num_splits = 1;
    L.grid = L.segs * L.num_splits;
    L.max_units = (int)((T + 31) / 32);
    L.max_portions = 1;
    L.slots = L.num_splits > 1 ? L.segs * L.num_splits : 0;
    return L;
  }
  long long g;
  if (split_tokens > 0) {
    const long long per = (split_tokens + 31) / 32;
    g = (L.units_max + per - 1) / per;
  } else {
    g = resident * L.waves;
  }
  if (g > L.units_max) g = L.units_max;
  if (g < 1) g = 1;
  long long mu = (L.units_max + g - 1) / g;
  if (mu > kMaxUnitsPerCta) {
    g = (L.units_max + kMaxUnitsPerCta - 1) / kMaxUnitsPerCta;
    mu = (L.units_max + g - 1) / g;
  }
  L.grid = g;
  L.max_units = (int)(mu < 1 ? 1 : mu);
  L.max_portions = (int)(L.segs < L.max_units ? L.segs : L.max_units);
  L.slots = L.segs + g;
  L.split_tokens = 32 * L.max_units;
  L.num_splits = 0;
  return L;
}

// FP8 tensor-core decode kernel.  rows_per_warp is 4, 8 or 16 and rbg (warps that
// share one K/V stream) 1, 2 or 4; stages 2 or 3.  1-D grid of `grid` CTAs
// (grid partition: segments x splits; balanced: one range each).
cudaError_t launch_decode_fp8(const DecodeParams& p, int rows_per_warp, int rbg, int stages,
                              long long grid, cudaStream_t stream);

// Tensor-core decode kernel (head_dim 128): 1-D grid of `grid` CTAs, one per
// (segment, split); stages = the K ring's depth, 2 or 3 (the V ring has 2).
cudaError_t launch_decode_tc(const DecodeParams& p, int stages, long long grid,
                             cudaStream_t stream);
size_t decode_tc_smem_bytes(int stages, int split_tokens, bool tok_scales);

// Dynamic shared memory of one decode CTA (rows = min(rows_per_cta, q_len * G)).
size_t decode_fp8_smem_bytes(int D, int stages, int rbg, int rows, int max_units,
                             int max_portions);

// Balanced partition without a split override: lower L.grid (and raise
// L.max_units) until the CTAs fill L.waves waves of resident CTAs on `sms`
// SMs, as far as the shared-memory footprint allows.  Needs a current CUDA
// device; leaves L alone if the occupancy query fails.
void decode_fp8_fit_grid(int D, int rows, int sms, DecodeLaunch& L);

// ------------------------------------------------------------ device helpers

#ifdef __CUDACC__

// A1, the order of the grid partition's work.  Its items are (sequence b,
// segment, split): a served sequence of length L has n = ceil(L / T) splits,
// and Hs segments (KV head x row block) each.  The items are ranked by a
// length key, largest first: every split of a sequence cut in n >= 2 splits
// counts as a whole split (ceil(T / 128) tiles), so that these sequences
// come first, segment-major (the splits of a segment neighbours: they end
// together and the segment's merge of its partials is not left for the end
// of the launch); a sequence served by one split ranks by its own number of
// 128-token tiles, so the shortest come last and fill the end of the launch.
// Ties by sequence.  Ranks past the last item (splits past a sequence's end)
// come last.  Every thread of the CTA calls it (it synchronises the CTA); it
// returns false when rank `ci` is past the last item, else the item.
// `served(bb, L)` says whether sequence bb of length L is served.  Shared
// memory: hist ceil(T / 128) + 1 ints, wsum one int per warp, res 4 ints.
template <int NTHREADS, class Served>
__device__ __forceinline__ bool longest_first_item(long long ci, int B,
                                                   const int32_t* __restrict__ seq_lens, int T,
                                                   int Hs, Served served, int* hist, int* wsum,
                                                   int* res, int& b, int& seg, int& split) {
  constexpr int NW = NTHREADS / 32;
  constexpr unsigned kAll = 0xFFFFFFFFu;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int TT = (T + 127) / 128;  // tiles of a whole split: the top key
  auto key_of = [&](int L, int n) { return n >= 2 ? TT : (L + 127) / 128; };
  for (int i = tid; i <= TT; i += NTHREADS) hist[i] = 0;
  __syncthreads();
  // sequences per key (each holds n x Hs items)
  long long top = 0;  // items of key TT
  for (int bb = tid; bb < B; bb += NTHREADS) {
    const int L = __ldg(seq_lens + bb);
    if (!served(bb, L)) continue;
    const int n = (L + T - 1) / T;
    const int k = key_of(L, n);
    if (k == TT)
      top += n;
    else
      atomicAdd(&hist[k], 1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) top += __shfl_xor_sync(kAll, top, o);
  if (lane == 0 && top > 0) atomicAdd(&hist[TT], (int)top);
  __syncthreads();
  // warp 0: the key (bin) of item rank ci and its rank within the bin,
  // scanning the bins from TT down, 32 at a time (bin counts in items)
  if (warp == 0) {
    long long base = 0, rank = 0;
    int bin = -1;
    for (int t0 = TT; t0 >= 1; t0 -= 32) {
      const int k = t0 - lane;
      const long long c = k >= 1 ? (long long)hist[k] * Hs : 0;
      long long incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long u = __shfl_up_sync(kAll, incl, o);
        if (lane >= o) incl += u;
      }
      const long long excl = base + incl - c;
      const unsigned hit = __ballot_sync(kAll, c > 0 && ci >= excl && ci < excl + c);
      if (bin < 0 && hit) {
        const int src = __ffs(hit) - 1;
        bin = __shfl_sync(kAll, k, src);
        rank = ci - __shfl_sync(kAll, excl, src);
      }
      base += __shfl_sync(kAll, incl, 31);
    }
    if (lane == 0) {
      res[0] = bin;
      res[1] = (int)rank;  // < B * n * Hs: the grid size, an int
      res[2] = -1;
    }
  }
  __syncthreads();
  const int bin = res[0], rank = res[1];
  if (bin < 0) return false;  // CTA-uniform
  // the rank-th item of the bin, in sequence order: sequence bb holds n x Hs
  // items of its key, segment-major
  long long done = 0;
  for (int b0 = 0; b0 < B && done <= rank; b0 += NTHREADS) {
    const int bb = b0 + tid;
    int c = 0, n = 0;
    if (bb < B) {
      const int L = __ldg(seq_lens + bb);
      if (served(bb, L)) {
        n = (L + T - 1) / T;
        c = key_of(L, n) == bin ? n : 0;
      }
    }
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(kAll, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const int x = wsum[w];
      before += w < warp ? x : 0;
      total += x;
    }
    // index among this sequence's items
    const long long j = rank - (done + (long long)(before + incl - c) * Hs);
    if (c > 0 && j >= 0 && j < (long long)c * Hs) {
      res[2] = bb;
      res[3] = (int)(j / n);  // segment
      res[0] = (int)(j % n);  // split
    }
    done += (long long)total * Hs;
    __syncthreads();  // wsum free for the next chunk; res written
  }
  b = res[2];
  seg = res[3];
  split = res[0];
  return b >= 0;  // both passes count the same items, so b >= 0 here
}

// f16x2 with `lo` in the low half.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Transpose an 8x8 matrix of 16-bit elements held one b32 pair per thread.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t r;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}

// Hardware base-2 exponential (ex2.approx); ex2(-inf) = +0.
__device__ __forceinline__ float fast_exp2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// ---- FP8 append helpers (shared by the append kernel and the fused decode)

// 16 consecutive inputs (f32 or bf16) starting at element `elem`, as exact f32.
__device__ __forceinline__ void load16_as_f32(const void* base, size_t elem, int dtype,
                                              float (&x)[16]) {
  if (dtype == ATLAS_DTYPE_F32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldg(p + i);
      x[4 * i + 0] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + elem);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint4 v = __ldg(p + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {  // bf16 -> f32 is exact: the bits move up 16
        x[8 * i + 2 * k + 0] = __uint_as_float(w[k] << 16);
        x[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
      }
    }
  }
}

// E4M3(fp32(x) / fp32(scale)): IEEE round-to-nearest division (never a
// reciprocal multiply), then round-to-nearest-even with saturation to +-448.
// Returns the 16 codes packed little-endian in 4 words.
__device__ __forceinline__ uint4 quantize16_e4m3(const float (&x)[16], float scale) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float y0 = __fdiv_rn(x[4 * i + 0], scale), y1 = __fdiv_rn(x[4 * i + 1], scale);
    const float y2 = __fdiv_rn(x[4 * i + 2], scale), y3 = __fdiv_rn(x[4 * i + 3], scale);
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(y0, y1), __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(y2, y3), __NV_SATFINITE, __NV_E4M3);
    w[i] = (lo & 0xFFFFu) | (hi << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// 16-byte chunk position of head dims [16j, 16j + 16) of K slot `slot`: with
// D = 128 each 128-byte token row is stored with its eight chunks permuted,
// chunk j at j XOR (slot % 8) -- the 128-byte swizzle of the tensor-core
// operand layout, so a 16-token piece copied verbatim into 1024-byte-aligned
// shared memory is a ready K-major operand; with D = 64 rows are plain.
__device__ __forceinline__ int k_chunk_pos(int D, int slot, int j) {
  return D == 128 ? (j ^ (slot & 7)) : j;
}

// Store 16 codes of head dims [16j, 16j + 16) of token slot `slot` of a head's
// page.  K pages are token-major [P][Hkv][ps][D] (chunks placed by
// k_chunk_pos); V pages are 16-slot groups, head-dim-major inside a group,
// [P][Hkv][ps/16][D][16], with slot t of a group at byte
// 4*((t%8)/2) + 2*(t/8) + t%2.
__device__ __forceinline__ void store16_k(uint8_t* k_pages, size_t head_page, int D, int ps,
                                          int slot, int j, uint4 codes) {
  uint8_t* dst = k_pages + (head_page * ps + slot) * D + 16 * k_chunk_pos(D, slot, j);
  *reinterpret_cast<uint4*>(dst) = codes;
}
__device__ __forceinline__ void store16_v(uint8_t* v_pages, size_t head_page, int D, int ps,
                                          int slot, int j, uint4 codes) {
  const int t = slot % 16;
  const int byte = 4 * ((t & 7) >> 1) + 2 * (t >> 3) + (t & 1);
  uint8_t* dst = v_pages + (head_page * (ps / 16) + slot / 16) * (16 * D) + (size_t)(16 * j) * 16 + byte;
  const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
#pragma unroll
  for (int k = 0; k < 16; ++k) dst[16 * k] = (uint8_t)(w[k >> 2] >> (8 * (k & 3)));
}

// ---- shared-memory addresses, mbarriers and bulk copies (single PTX instructions)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Orders this thread's earlier global writes before later async-proxy reads.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// One bounded probe of an mbarrier phase; the thread may sleep up to
// ~0.5 ms inside the instruction while the phase is still pending.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(500000u)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// This SM's cycle counter.  Bounded waits measure with it rather than with
// the global nanosecond timer, which is far slower to read: a wait loop that
// reads that timer on every pass delays the hand-offs it waits for.
__device__ __forceinline__ uint64_t sm_cycles() { return (uint64_t)clock64(); }

// A wait limit in nanoseconds as SM cycles, at two cycles per nanosecond: at
// least the limit at any SM clock up to 2 GHz (a slower clock only stretches
// it).
__device__ __forceinline__ uint64_t ns_to_cycles(uint64_t ns) { return 2 * ns; }

// Wait for an mbarrier phase with a time limit; false if it ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = sm_cycles(), limit = ns_to_cycles(limit_ns);
  while (!mbar_try_wait(bar, parity)) {
    if (sm_cycles() - t0 > limit) return false;
  }
  return true;
}

// 1-D bulk copy global -> shared of `bytes` (multiple of 16, both addresses
// 16-byte aligned), completion counted on `bar` (no multicast).  The KV pages
// are read once per call: the L2 lines they fill are marked evict-first.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
  return policy;
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  bulk_load(dst, src, bytes, bar, l2_evict_first_policy());
}

#endif  // __CUDACC__

}  // namespace atlas
