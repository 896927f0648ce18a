// Decode / MTP-verify attention without any device allocation by the caller.
//
// Some callers cannot allocate device memory for a workspace: code that runs
// inside a host framework which owns every allocation (a plugin, an embedded
// runtime handed only input and output buffers), or a code path that must not
// touch the allocator at all.  For them, atlas_paged_gqa_decode_noalloc runs
// the same decode kernel as atlas_paged_gqa_decode but keeps its scratch --
// the split-KV partial results, the per-(sequence, KV head, row group)
// completion counters and the device error word -- in one file-scope
// __device__ array of kScratchBytes bytes.  Every GPU that loads the library
// holds that array until the process exits.  Nothing here calls cudaMalloc,
// cudaFree or any allocating routine.
//
// The array is shared by every call on a device and keeps the last call's
// contents; each call clears the counters and the error word (the only parts
// that must start at zero) with cudaMemsetAsync on its stream before the
// launch.  Calls whose kernels overlap on the GPU (different streams, no
// ordering) race on the array.  If the split-KV partials of a call would not
// fit, the call uses longer splits (down to one split per sequence); a call
// whose counters alone would not fit, or that would need splits longer than
// 65536 tokens, is rejected with ATLAS_ERR_WORKSPACE.
// The first call on a device looks up the array's device address
// (cudaGetSymbolAddress) with that device current; make that first call
// before any stream capture.  Device-side checks still zero the rows of an
// invalid sequence and skip bad page ids, but this variant has no error word
// the caller can read.
#include <math.h>

#include <mutex>

#include "atlas_internal.cuh"

namespace {

constexpr size_t kScratchBytes = 8u << 20;  // 8 MiB per GPU
constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_decode_scratch[kScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up once).
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = ptr;
  }
  return g_scratch_addr[dev];
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) % 16) == 0; }

}  // namespace

extern "C" atlas_status_t atlas_paged_gqa_decode_noalloc(
    const void* q, const void* k_pages, const void* v_pages, const float* k_scale,
    const float* v_scale, const int32_t* block_table, int32_t max_blocks_per_seq,
    const int32_t* seq_lens, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t page_size, int32_t num_pages, int32_t q_len, int32_t max_seq_len,
    float sm_scale, void* out, void* stream) {
  if (batch < 0 || num_kv_heads < 1 || num_q_heads < 1 || num_q_heads % num_kv_heads != 0 ||
      q_len < 1 || num_pages < 1 || max_blocks_per_seq < 1 || max_seq_len < q_len)
    return ATLAS_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return ATLAS_ERR_UNSUPPORTED;
  if (page_size < 16 || page_size > 1024 || page_size % 16 != 0) return ATLAS_ERR_UNSUPPORTED;
  if ((long long)max_seq_len > (long long)max_blocks_per_seq * page_size) return ATLAS_ERR_INVALID_ARG;
  if (!(sm_scale == sm_scale) || isinf(sm_scale)) return ATLAS_ERR_INVALID_ARG;
  if (batch == 0) return ATLAS_OK;
  if (!q || !k_pages || !v_pages || !k_scale || !v_scale || !block_table || !seq_lens || !out)
    return ATLAS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_pages) || !aligned16(v_pages))
    return ATLAS_ERR_INVALID_ARG;
  if (batch > 65535 || num_kv_heads > 65535) return ATLAS_ERR_UNSUPPORTED;

  // launch shape: the same choice of rows per warp / warps per K/V stream as
  // the pool-based entry point
  const int G = num_q_heads / num_kv_heads;
  const int R = q_len * G;
  const int rows_per_warp = (R <= 8) ? 8 : 16;
  const int rbg = (R <= 16) ? 1 : (R <= 32 ? 2 : 4);
  const int rows_per_cta = rows_per_warp * rbg;
  const int row_blocks = (R + rows_per_cta - 1) / rows_per_cta;
  const int stages = (rbg == 1) ? 2 : 3;
  const int rows_all = q_len * num_q_heads;

  // scratch layout: [error word][counters][log2-sum-exp][O partials]
  const size_t counters_bytes =
      align_up((size_t)batch * num_kv_heads * row_blocks * sizeof(int32_t), kAlign);
  if (kAlign + counters_bytes > kScratchBytes) return ATLAS_ERR_WORKSPACE;
  const size_t room = kScratchBytes - kAlign - counters_bytes;
  const size_t per_split = (size_t)batch * rows_all * (head_dim + 1) * sizeof(float) + 2 * kAlign;

  // split size: about two waves of 4 resident CTAs per SM if every sequence
  // were max_seq_len long, 256..8192 tokens, then lengthened until the
  // partials fit in the scratch
  int sms = 148;
  {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
      sms = n;
  }
  const long long units = (long long)batch * num_kv_heads * row_blocks;
  long long want = ((long long)sms * 8 + units - 1) / units;
  if (want < 1) want = 1;
  long long T = (max_seq_len + want - 1) / want;
  T = (T + 63) / 64 * 64;
  if (T < 256) T = 256;
  if (T > 8192) T = 8192;
  int num_splits = (int)((max_seq_len + T - 1) / T);
  if (num_splits > 1 && (size_t)num_splits * per_split > room) {
    const long long fit = (long long)(room / per_split);
    if (fit <= 1) {
      num_splits = 1;
      T = ((long long)max_seq_len + 63) / 64 * 64;
    } else {
      T = ((max_seq_len + fit - 1) / fit + 63) / 64 * 64;
      num_splits = (int)((max_seq_len + T - 1) / T);
    }
  }
  if (num_splits == 1 && T < max_seq_len) T = ((long long)max_seq_len + 63) / 64 * 64;
  // one split holds its page-piece table in shared memory: bound its length
  if (T > 65536) return ATLAS_ERR_WORKSPACE;

  uint8_t* scratch = static_cast<uint8_t*>(scratch_on_current_device());
  if (!scratch) return ATLAS_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, kAlign + counters_bytes, s) != cudaSuccess) return ATLAS_ERR_CUDA;

  atlas::DecodeParams p{};  // value-initialised: no fused append unless set
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_pages = static_cast<const uint8_t*>(k_pages);
  p.v_pages = static_cast<const uint8_t*>(v_pages);
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.err = reinterpret_cast<int32_t*>(scratch);
  p.counters = reinterpret_cast<int32_t*>(scratch + kAlign);
  const size_t lse_bytes = align_up((size_t)batch * num_splits * rows_all * sizeof(float), kAlign);
  p.part_lse = reinterpret_cast<float*>(scratch + kAlign + counters_bytes);
  p.part_o = reinterpret_cast<float*>(scratch + kAlign + counters_bytes + lse_bytes);
  p.B = batch;
  p.Hq = num_q_heads;
  p.Hkv = num_kv_heads;
  p.G = G;
  p.q_len = q_len;
  p.D = head_dim;
  p.ps = page_size;
  p.num_pages = num_pages;
  p.max_blocks = max_blocks_per_seq;
  p.split_tokens = (int)T;
  p.num_splits = num_splits;
  p.row_blocks = row_blocks;
  const double scale = sm_scale > 0.f ? (double)sm_scale : 1.0 / sqrt((double)head_dim);
  p.qk_scale_log2 = (float)(scale * 1.4426950408889634);  // log2(e)
  p.k_new = nullptr;  // decode only
  p.v_new = nullptr;
  cudaError_t e = atlas::launch_decode_fp8(p, rows_per_warp, rbg, stages, s);
  return e == cudaSuccess ? ATLAS_OK : ATLAS_ERR_CUDA;
}
