// FP8 page append: quantise new K/V rows to E4M3 with a per-KV-head scale and
// scatter them into their pages through the block table.
//
// Source: the FP8 KV quantisation with scale factors of the Atlas deep-dive
// (ainews.cool, "Quantisation" paragraph) and the paged FP8 KV cache of the
// GB10 page (ainews.surl.tw).  Encoding reading: y = fp32(x) / fp32(scale[h])
// as an IEEE round-to-nearest division (__fdiv_rn, never a reciprocal
// multiply), then round-to-nearest-even to E4M3 with saturation to +-448
// (cvt.rn.satfinite), sign of zero kept.  The result must be bit-exact with
// that definition.
//
// Finer-grained mode (k_tok_scale != nullptr): each token's row of each KV
// head gets its own dynamic scale amax / 448, stored at [page][head][slot] of
// the scale arrays, and the head's bound of the V scales is raised to it.
//
// Page layouts: K pages are token-major [P][Hkv][ps][D] (with D = 128 the
// 16-byte chunk j of slot s sits at chunk position j XOR (s % 8)); V pages are kept in
// groups of 16 slots, head-dim-major inside a group: [P][Hkv][ps/16][D][16]
// (16 consecutive tokens of one head dimension adjacent), slot t of a group at
// byte 4*((t%8)/2) + 2*(t/8) + t%2 (bytes 4c..4c+3 hold slots 2c, 2c+1, 2c+8,
// 2c+9, the token order of the decode kernel's P fragments).
// Memory-bound: per element 4 (f32) or 2 (bf16) bytes read, 1 byte written.
// A CTA owns 16 consecutive new tokens of one (sequence, KV head), D threads.
// K: thread (token, chunk) quantises 16 consecutive elements of one token row
// and stores them as one 16-byte write.  V: thread d takes head dimension d of
// the 16 tokens (every load instruction reads one token row across the CTA,
// coalesced), so the group row of dimension d -- 16 codes in the group's slot
// order -- is formed in registers and leaves as one 16-byte write when the 16
// tokens fill one 16-slot group of a page exactly (the cache-fill case); the
// few tokens of a decode step are stored as single bytes.
#include "atlas_internal.cuh"

namespace atlas {
namespace {

constexpr int kTok = 16;  // tokens per CTA (one 16-slot V group when aligned)

// Dynamic per-(token, KV head) scale of the finer-grained mode: the largest
// |x| over the token's D elements (held 16 per thread by the CH = D / 16
// consecutive threads of the token), divided by 448 (IEEE division); 1 for an
// all-zero row.  Every thread of the warp takes part in the shuffles.
template <int CH>
__device__ __forceinline__ float token_row_scale(const float (&x)[16]) {
  float a = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) a = fmaxf(a, fabsf(x[k]));
#pragma unroll
  for (int o = 1; o < CH; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  return a > 0.f ? __fdiv_rn(a, 448.f) : 1.f;
}

template <int D, bool TS>
__global__ void __launch_bounds__(D) fp8_append_kernel(const AppendParams p) {
  constexpr int CH = D / 16;  // 16-element chunks per row
  __shared__ int s_page[kTok];
  const int n_tiles = (p.n_new + kTok - 1) / kTok;
  const int tile = blockIdx.x % n_tiles;
  const int bh = blockIdx.x / n_tiles;
  const int h = bh % p.Hkv, b = bh / p.Hkv;
  const int t0 = tile * kTok;
  const int n_tok = min(kTok, p.n_new - t0);
  const int start = __ldg(p.start_pos + b);
  const int tid = threadIdx.x;
  const int lt = tid / CH, j = tid % CH;  // K: token within the tile, chunk

  if (tid < kTok) {  // page of each token of the tile (-1: not written, flagged)
    int page = -1;
    const int pos = start + t0 + tid;
    if (tid < n_tok) {
      const int blk = pos / p.ps;
      if (pos >= 0 && blk < p.max_blocks) {
        page = __ldg(p.block_table + (size_t)b * p.max_blocks + blk);
        if (page < 0 || page >= p.num_pages) page = -1;
      }
      if (page < 0) atomicOr(p.err, ATLAS_DEVERR_APPEND);
    }
    s_page[tid] = page;
  }

  // ---- V: thread (q, c) = (tid / (D/4), tid % (D/4)) loads head dims
  // 4c .. 4c + 3 of the four tokens 2q, 2q + 1, 2q + 8, 2q + 9 (one 16-byte
  // load per token for f32, 8 bytes for bf16): exactly the four slots that
  // share word q of a 16-slot group row, so each of its four dims yields one
  // 32-bit word.  The words meet in shared memory ([d][16 slots], the group
  // row layout) and thread d stores its dimension's row -- one 16-byte write
  // when the 16 tokens fill one group of one page (the cache-fill case),
  // single bytes otherwise (a decode step's few tokens).
  constexpr int C4 = D / 4;
  const int vq = tid / C4, vc = tid % C4;
  int vt[4];
  vt[0] = 2 * vq;
  vt[1] = 2 * vq + 1;
  vt[2] = 2 * vq + 8;
  vt[3] = 2 * vq + 9;
  float xv[4][4];  // [token k of the four][dim e]
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int t = vt[k];
#pragma unroll
    for (int e = 0; e < 4; ++e) xv[k][e] = 0.f;
    if (t < n_tok) {
      const size_t el = (((size_t)b * p.n_new + t0 + t) * p.Hkv + h) * D + 4 * vc;
      if (p.dtype == ATLAS_DTYPE_F32) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(p.v_new) + el));
        xv[k][0] = f.x; xv[k][1] = f.y; xv[k][2] = f.z; xv[k][3] = f.w;
      } else {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(
            static_cast<const __nv_bfloat16*>(p.v_new) + el));
        xv[k][0] = __uint_as_float(w.x << 16); xv[k][1] = __uint_as_float(w.x & 0xFFFF0000u);
        xv[k][2] = __uint_as_float(w.y << 16); xv[k][3] = __uint_as_float(w.y & 0xFFFF0000u);
      }
    }
  }
  float vsc[4];  // the four tokens' V scales
  if constexpr (TS) {
    // per-token scales: the token's row maximum over all D dims -- the C4
    // threads of one q hold the row (one warp at D = 128, half a warp at 64)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float a = fmaxf(fmaxf(fabsf(xv[k][0]), fabsf(xv[k][1])), fmaxf(fabsf(xv[k][2]), fabsf(xv[k][3])));
#pragma unroll
      for (int o = C4 / 2; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
      vsc[k] = a > 0.f ? __fdiv_rn(a, 448.f) : 1.f;
    }
  } else {
    const float s0 = __ldg(p.v_scale + h);
#pragma unroll
    for (int k = 0; k < 4; ++k) vsc[k] = s0;
  }
  __shared__ __align__(16) uint32_t s_v[D][4];  // [d][word]: group row of dim d
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    // word q of dim 4c + e: bytes = slots 2q, 2q + 1, 2q + 8, 2q + 9
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(xv[0][e], vsc[0]), __fdiv_rn(xv[1][e], vsc[1])), __NV_SATFINITE,
        __NV_E4M3);
    const uint32_t hi2 = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(xv[2][e], vsc[2]), __fdiv_rn(xv[3][e], vsc[3])), __NV_SATFINITE,
        __NV_E4M3);
    s_v[4 * vc + e][vq] = (lo & 0xFFFFu) | ((hi2 & 0xFFFFu) << 16);
  }
  __syncthreads();  // the group rows (and s_page) are complete
  if (TS && vc == 0) {  // the four tokens' V scales and the head's bound
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int t = vt[k];
      if (t >= n_tok || s_page[t] < 0) continue;
      const int slot = (start + t0 + t) % p.ps;
      p.v_tok_scale[((size_t)s_page[t] * p.Hkv + h) * p.ps + slot] = vsc[k];
      // positive floats order like their bit patterns: the head's running
      // bound of the per-token V scales
      atomicMax(reinterpret_cast<int*>(p.v_scale_bound + h), __float_as_int(vsc[k]));
    }
  }
  const int p0 = start + t0;
  const bool whole_group = n_tok == kTok && (p0 % 16) == 0 && s_page[0] >= 0;
  {
    const int d = tid;  // this thread's dimension: its 16 codes in group order
    const uint4 row = *reinterpret_cast<const uint4*>(&s_v[d][0]);
    if (whole_group) {
      const size_t head_page = (size_t)s_page[0] * p.Hkv + h;
      uint8_t* dst = p.v_pages + (head_page * (p.ps / 16) + (p0 % p.ps) / 16) * (16 * D) + 16 * d;
      *reinterpret_cast<uint4*>(dst) = row;
    } else {  // byte stores for the valid tokens (a decode step's few tokens)
      const uint32_t rw[4] = {row.x, row.y, row.z, row.w};
#pragma unroll
      for (int t = 0; t < kTok; ++t) {
        const int pg = s_page[t];
        if (t >= n_tok || pg < 0) continue;
        const int slot = (p0 + t) % p.ps;
        const int g = slot % 16;
        const int byte = 4 * ((g & 7) >> 1) + 2 * (g >> 3) + (g & 1);
        const int tb = 4 * ((t & 7) >> 1) + 2 * (t >> 3) + (t & 1);  // token t in the row
        const size_t head_page = (size_t)pg * p.Hkv + h;
        p.v_pages[(head_page * (p.ps / 16) + slot / 16) * (16 * D) + 16 * d + byte] =
            (uint8_t)(rw[tb >> 2] >> (8 * (tb & 3)));
      }
    }
  }

  // ---- K, 16 consecutive elements of one token row per thread (one
  // 16-byte store of codes each)
  const int pos = start + t0 + lt;
  const int page = s_page[lt];
  const bool ok = lt < n_tok && page >= 0;
  float x[16];
  if (ok) {
    load16_as_f32(p.k_new, (((size_t)b * p.n_new + t0 + lt) * p.Hkv + h) * D + 16 * j, p.dtype,
                  x);
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) x[k] = 0.f;
  }
  const float ks = TS ? token_row_scale<CH>(x) : __ldg(p.k_scale + h);
  if (ok) {
    const size_t head_page = (size_t)page * p.Hkv + h;
    const int slot = pos % p.ps;
    store16_k(p.k_pages, head_page, D, p.ps, slot, j, quantize16_e4m3(x, ks));
    if (TS && j == 0) p.k_tok_scale[head_page * p.ps + slot] = ks;
  }
}

}  // namespace

cudaError_t launch_fp8_append(const AppendParams& p, int num_sms, cudaStream_t stream) {
  (void)num_sms;
  if (p.batch == 0 || p.n_new == 0) return cudaSuccess;
  const long long n_tiles = (p.n_new + kTok - 1) / kTok;
  const long long blocks = n_tiles * p.Hkv * p.batch;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const bool ts = p.k_tok_scale != nullptr;
  if (p.D == 128) {
    if (ts)
      fp8_append_kernel<128, true><<<(unsigned)blocks, 128, 0, stream>>>(p);
    else
      fp8_append_kernel<128, false><<<(unsigned)blocks, 128, 0, stream>>>(p);
  } else if (p.D == 64) {
    if (ts)
      fp8_append_kernel<64, true><<<(unsigned)blocks, 64, 0, stream>>>(p);
    else
      fp8_append_kernel<64, false><<<(unsigned)blocks, 64, 0, stream>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace atlas
