// C ABI of the paged-KV-cache decode library: argument checks, launch
// configuration, tensor-map encoding and kernel launches.  Every kernel of
// the library is compiled in this one translation unit (the device error word
// in pa_device.cuh is defined once).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <mutex>

#include "pa.h"
#include "pa_device.cuh"
#include "cache_ops.cuh"
#include "decode_attention.cuh"
#include "prefill_attention.cuh"

namespace {

constexpr int kWarpsPerCta = 4;
constexpr int kMaxDevices = 64;
constexpr int kMaxCtasPerSm = 4;

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int sm_count(int dev) {
  static std::atomic<int> cache[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return 0;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Limit of every bounded wait on an asynchronous copy or MMA in the kernels
// launched from now on (pa_set_wait_limit).
constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;   // 2 s
std::atomic<unsigned long long> g_wait_limit_ns{kDefaultWaitLimitNs};

// User overrides of the launch heuristics (0 = automatic).
std::atomic<int> g_tune_nstage{0};
std::atomic<int> g_tune_ctas{0};
std::atomic<int> g_tune_min_tiles{0};

struct DecodeLayout {
  int nstage, ctas_per_sm, grid, w_total, min_tiles;
  size_t smem;
  size_t off_meta, off_ml, off_o, workspace;
};

size_t stage_bytes(int D, int B, int G) {
  return 2 * (size_t)B * D * 2 + (size_t)G * D * 2 + 4 * (size_t)D + sizeof(pa::TileInfo) +
         sizeof(uint64_t);
}

// Shared-memory need of one CTA with `nstage` stages per warp.
size_t cta_smem(int D, int B, int G, int nstage) {
  return 1024 + (size_t)kWarpsPerCta * nstage * stage_bytes(D, B, G);
}

size_t workspace_for(int w_total, int G, int D, size_t *off_ml, size_t *off_o) {
  size_t meta = round_up((size_t)w_total * pa::kMetaWords * sizeof(long long), 256);
  size_t ml = round_up((size_t)2 * w_total * G * 2 * sizeof(float), 256);
  size_t o = round_up((size_t)2 * w_total * G * D * sizeof(float), 256);
  if (off_ml) *off_ml = meta;
  if (off_o) *off_o = meta + ml;
  return meta + ml + o;
}

// CTAs per SM and stages per warp.  Each warp issues its own copies, so
// resident warps are what keeps HBM busy; measured on B200, two stages per
// warp with the most CTAs per SM beat deeper rings with fewer warps for every
// workload shape (even one stage with twice the warps beat three stages).
// So: the most CTAs per SM (at most 3) that registers and shared memory allow
// with at least one stage, and up to two stages per warp.
void choose_layout(int D, int B, int G, int sms, int regs_per_thread, DecodeLayout *L) {
  const size_t per_sm = 228 * 1024;   // shared memory per SM
  const size_t per_cta_reserved = 1024;
  const size_t set = (size_t)kWarpsPerCta * stage_bytes(D, B, G);
  const int want_ctas = g_tune_ctas.load();
  const int want_stages = g_tune_nstage.load();
  int reg_ctas = regs_per_thread > 0 ? 65536 / (regs_per_thread * kWarpsPerCta * 32) : 2;
  reg_ctas = std::max(1, std::min(reg_ctas, 3));
  auto stages_for = [&](int c) {
    const size_t budget = per_sm / c - per_cta_reserved - 256;   // 256: static smem
    return (int)((budget - 1024) / set);
  };
  // Every warp streams through its own ring, so the tiles in flight per SM,
  // CTAs x stages (stages at most 2), are what keep HBM busy: take the most,
  // and on a tie the layout with more stages, whose warps overlap a copy with
  // the math (measured on B200 at block 32, 64 q / 8 kv heads: 1 CTA x 2
  // stages beats 2 CTAs x 1 stage by ~1 %).
  int ctas = 1, best = 0, best_st = 0;
  for (int c = reg_ctas; c >= 1; --c) {
    const int st = std::min(stages_for(c), 2);
    if (st < 1) continue;
    if (c * st > best || (c * st == best && st > best_st)) {
      best = c * st;
      best_st = st;
      ctas = c;
    }
  }
  if (want_ctas > 0) ctas = std::min(want_ctas, kMaxCtasPerSm);
  int nst = std::min(stages_for(ctas), 2);
  if (want_stages > 0) nst = std::min(stages_for(ctas), want_stages);
  nst = std::max(nst, 1);
  L->nstage = nst;
  L->ctas_per_sm = ctas;
  L->grid = sms * ctas;
  L->w_total = L->grid * kWarpsPerCta;
  const int mt = g_tune_min_tiles.load();
  L->min_tiles = mt > 0 ? mt : 4;
  L->smem = cta_smem(D, B, G, nst);
  L->off_meta = 0;
  L->workspace = workspace_for(L->w_total, G, D, &L->off_ml, &L->off_o);
}

bool encode_pool_map(CUtensorMap *m, const void *base, long long rows, int D, int B) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)B};
  cuuint32_t estr[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DecodeArgs {
  float *out;
  const void *q, *k_cache, *v_cache;
  const void *k_new, *v_new;   // non-null: fused decode step (cache write of the newest token)
  const int32_t *block_tables, *context_lens;
  float scale;
  int num_kv_heads, num_seqs, num_q_heads, head_dim, block_size, max_blocks, num_blocks;
  void *workspace;
  size_t workspace_bytes;
  cudaStream_t stream;
};

template <typename T, int D, int B, int NT>
int launch_decode(const DecodeArgs &a, int dev, int sms) {
  const int G = a.num_q_heads / a.num_kv_heads;
  auto kern = pa::paged_decode_kernel<T, D, B, NT, kWarpsPerCta>;
  static std::atomic<int> regs_cache{0};
  int regs = regs_cache.load();
  if (regs == 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return PA_ERR_CUDA;
    regs = fa.numRegs;
    regs_cache.store(regs);
  }
  DecodeLayout L;
  choose_layout(D, B, G, sms, regs, &L);
  if (a.workspace_bytes < L.workspace) return PA_ERR_WORKSPACE;

  static std::atomic<size_t> attr_set[kMaxDevices];
  if (attr_set[dev].load() < L.smem) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.smem) !=
        cudaSuccess)
      return PA_ERR_CUDA;
    attr_set[dev].store(L.smem);
  }
  CUtensorMap kmap, vmap;
  const long long rows = (long long)a.num_blocks * a.num_kv_heads * B;
  if (!encode_pool_map(&kmap, a.k_cache, rows, D, B) ||
      !encode_pool_map(&vmap, a.v_cache, rows, D, B))
    return PA_ERR_CUDA;

  uint8_t *ws = static_cast<uint8_t *>(a.workspace);
  pa::DecodeParams p;
  p.out = a.out;
  p.q = static_cast<const uint8_t *>(a.q);
  p.k_new = static_cast<const uint8_t *>(a.k_new);
  p.v_new = static_cast<const uint8_t *>(a.v_new);
  p.k_cache_w = static_cast<uint8_t *>(const_cast<void *>(a.k_cache));
  p.v_cache_w = static_cast<uint8_t *>(const_cast<void *>(a.v_cache));
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  p.meta = reinterpret_cast<long long *>(ws + L.off_meta);
  p.part_ml = reinterpret_cast<float *>(ws + L.off_ml);
  p.part_o = reinterpret_cast<float *>(ws + L.off_o);
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.num_seqs = a.num_seqs;
  p.num_q_heads = a.num_q_heads;
  p.num_kv_heads = a.num_kv_heads;
  p.group = G;
  p.head_dim = D;
  p.max_blocks = a.max_blocks;
  p.num_blocks = a.num_blocks;
  p.nstage = L.nstage;
  p.min_tiles = L.min_tiles;
  p.wait_ns = g_wait_limit_ns.load();

  // Programmatic dependent launch: the grid may be scheduled while the
  // previous kernel on the stream (typically reshape_and_cache) is still
  // running; the kernel waits for it (griddepcontrol.wait) before its first
  // global-memory read.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.grid);
  cfg.blockDim = dim3(kWarpsPerCta * 32);
  cfg.dynamicSmemBytes = L.smem;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, kmap, vmap, p) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  // Split merge: one warp per (boundary between warp ranges, group of up to
  // four heads, two when the group is larger), resident and waiting before
  // the streaming grid completes.
  if (L.w_total > 1) {
    cudaLaunchConfig_t mc = {};
    mc.blockDim = dim3(128);
    mc.dynamicSmemBytes = 0;
    mc.stream = a.stream;
    mc.attrs = attr;
    mc.numAttrs = 1;
    cudaError_t e;
    if (G <= 4) {
      mc.gridDim = dim3((unsigned)((L.w_total - 1 + 3) / 4));
      e = cudaLaunchKernelEx(&mc, pa::paged_decode_merge_kernel<D, 4>, p, L.w_total, 1);
    } else {
      const int hc = (G + 1) / 2;
      mc.gridDim = dim3((unsigned)(((long long)(L.w_total - 1) * hc + 3) / 4));
      e = cudaLaunchKernelEx(&mc, pa::paged_decode_merge_kernel<D, 2>, p, L.w_total, hc);
    }
    if (e != cudaSuccess) {
      cudaGetLastError();
      return PA_ERR_CUDA;
    }
  }
  return PA_OK;
}

template <typename T, int D, int B>
int dispatch_group(const DecodeArgs &a, int dev, int sms) {
  const int G = a.num_q_heads / a.num_kv_heads;
  if (G == 1) return launch_decode<T, D, B, 0>(a, dev, sms);
  if (G <= 8) return launch_decode<T, D, B, 1>(a, dev, sms);
  return launch_decode<T, D, B, 2>(a, dev, sms);
}

template <typename T>
int dispatch_shape(const DecodeArgs &a, int dev, int sms) {
  if (a.head_dim == 128 && a.block_size == 16) return dispatch_group<T, 128, 16>(a, dev, sms);
  if (a.head_dim == 128 && a.block_size == 32) return dispatch_group<T, 128, 32>(a, dev, sms);
  if (a.head_dim == 64 && a.block_size == 16) return dispatch_group<T, 64, 16>(a, dev, sms);
  return dispatch_group<T, 64, 32>(a, dev, sms);
}

// ---------------------------------------------------------------- chunked prefill

#include "prefill_launch.cuh"

bool supported_shape(int head_dim, int block_size) {
  return (head_dim == 64 || head_dim == 128) && (block_size == 16 || block_size == 32);
}

int current_device(int *dev) { return cudaGetDevice(dev) == cudaSuccess ? PA_OK : PA_ERR_CUDA; }

}  // namespace

// ---------------------------------------------------------------------------
// Scratch for pa_paged_decode_attention_no_alloc: a fixed array in device
// global memory, part of the library's module, so that entry point needs no
// allocation.  Every GPU that loads the library holds these bytes until the
// process exits.  In host code the name is only a stand-in for the device
// array: its device address comes from cudaGetSymbolAddress, once per device.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // PA_NO_ALLOC_SCRATCH_BYTES
static __device__ __align__(256) unsigned char g_no_alloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of g_no_alloc_scratch on the current device `dev`, looked up
// on the first call for that device (which must therefore not be inside a
// stream capture) and cached.
int no_alloc_scratch(int dev, void **out) {
  static std::mutex mu;
  static void *ptrs[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_no_alloc_scratch) != cudaSuccess || p == nullptr)
      return PA_ERR_CUDA;
    ptrs[dev] = p;
  }
  *out = ptrs[dev];
  return PA_OK;
}

}  // namespace

extern "C" {

const char *pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_ARG: return "PA_ERR_ARG: invalid argument";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: shape not implemented";
    case PA_ERR_NO_BLOCKS: return "PA_ERR_NO_BLOCKS: free list exhausted";
    case PA_ERR_SEQ: return "PA_ERR_SEQ: unknown or duplicate sequence";
    case PA_ERR_CUDA: return "PA_ERR_CUDA: CUDA runtime call failed";
    case PA_ERR_DEVICE_BOUNDS: return "PA_ERR_DEVICE_BOUNDS: device-side index check fired";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE: workspace too small or misaligned";
    default: return "unknown pa_status";
  }
}

int pa_version(void) { return 100; }

int pa_reshape_and_cache(const void *key, const void *value, void *k_cache, void *v_cache,
                         const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                         pa_stream_t stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks < 0 || head_dim <= 0 || block_size <= 0)
    return PA_ERR_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_ARG;
  if (!supported_shape(head_dim, block_size)) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_ARG;
  if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(slot_mapping, 8))
    return PA_ERR_ARG;
  const int vec_per_row = head_dim * 2 / 16;
  const long long num_vec = (long long)num_tokens * num_kv_heads * vec_per_row;
  const long long blocks = std::min<long long>((num_vec + 255) / 256, 1 << 20);
  pa::reshape_and_cache_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(
      static_cast<const uint4 *>(key), static_cast<const uint4 *>(value),
      static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), slot_mapping, num_vec,
      vec_per_row, num_kv_heads, block_size, (long long)num_blocks * block_size);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

size_t pa_paged_decode_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads,
                                       int head_dim, int block_size, int max_context_len) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_context_len < 0) return 0;
  if (num_q_heads % num_kv_heads != 0 || num_q_heads / num_kv_heads > 16) return 0;
  if (!supported_shape(head_dim, block_size)) return 0;
  int dev;
  if (current_device(&dev) != PA_OK) return 0;
  const int sms = sm_count(dev);
  if (sms <= 0) return 0;
  const int G = num_q_heads / num_kv_heads;
  return workspace_for(sms * kWarpsPerCta * kMaxCtasPerSm, G, head_dim, nullptr, nullptr);
}

int pa_paged_decode_attention(float *out, const void *q, const void *k_cache,
                              const void *v_cache, const int32_t *block_tables,
                              const int32_t *context_lens, float scale, int num_kv_heads,
                              int num_seqs, int num_q_heads, int head_dim, int block_size,
                              int max_blocks_per_seq, int max_context_len, int num_blocks,
                              pa_dtype dtype, void *workspace, size_t workspace_bytes,
                              pa_stream_t stream) {
  if (num_seqs < 0 || num_kv_heads <= 0 || num_q_heads <= 0 || head_dim <= 0 || block_size <= 0)
    return PA_ERR_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_ARG;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_ARG;
  if (!supported_shape(head_dim, block_size) || num_q_heads / num_kv_heads > 16)
    return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (max_blocks_per_seq <= 0 || num_blocks <= 0 || max_context_len < 0 ||
      (long long)max_context_len > (long long)max_blocks_per_seq * block_size)
    return PA_ERR_ARG;
  if ((long long)num_blocks * num_kv_heads * block_size >= (1ll << 31)) return PA_ERR_UNSUPPORTED;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PA_ERR_ARG;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return PA_ERR_ARG;
  if (!workspace || !aligned(workspace, 256)) return PA_ERR_WORKSPACE;
  int dev;
  if (current_device(&dev) != PA_OK || dev >= kMaxDevices) return PA_ERR_CUDA;
  const int sms = sm_count(dev);
  if (sms <= 0) return PA_ERR_CUDA;
  DecodeArgs a{out,          q,           k_cache,      v_cache,      nullptr,
               nullptr,      block_tables, context_lens, scale,        num_kv_heads,
               num_seqs,     num_q_heads, head_dim,     block_size,   max_blocks_per_seq,
               num_blocks,   workspace,   workspace_bytes, (cudaStream_t)stream};
  if (dtype == PA_BF16) return dispatch_shape<__nv_bfloat16>(a, dev, sms);
  return dispatch_shape<__half>(a, dev, sms);
}

int pa_decode_step(float *out, const void *q, const void *k_new, const void *v_new,
                   void *k_cache, void *v_cache, const int32_t *block_tables,
                   const int32_t *context_lens, float scale, int num_kv_heads, int num_seqs,
                   int num_q_heads, int head_dim, int block_size, int max_blocks_per_seq,
                   int max_context_len, int num_blocks, pa_dtype dtype, void *workspace,
                   size_t workspace_bytes, pa_stream_t stream) {
  if (num_seqs < 0 || num_kv_heads <= 0 || num_q_heads <= 0 || head_dim <= 0 || block_size <= 0)
    return PA_ERR_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_ARG;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_ARG;
  if (!supported_shape(head_dim, block_size) || num_q_heads / num_kv_heads > 16)
    return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (max_blocks_per_seq <= 0 || num_blocks <= 0 || max_context_len < 0 ||
      (long long)max_context_len > (long long)max_blocks_per_seq * block_size)
    return PA_ERR_ARG;
  if ((long long)num_blocks * num_kv_heads * block_size >= (1ll << 31)) return PA_ERR_UNSUPPORTED;
  if (!out || !q || !k_new || !v_new || !k_cache || !v_cache || !block_tables || !context_lens)
    return PA_ERR_ARG;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) ||
      !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(block_tables, 4) ||
      !aligned(context_lens, 4))
    return PA_ERR_ARG;
  if (!workspace || !aligned(workspace, 256)) return PA_ERR_WORKSPACE;
  int dev;
  if (current_device(&dev) != PA_OK || dev >= kMaxDevices) return PA_ERR_CUDA;
  const int sms = sm_count(dev);
  if (sms <= 0) return PA_ERR_CUDA;
  DecodeArgs a{out,          q,           k_cache,      v_cache,      k_new,
               v_new,        block_tables, context_lens, scale,        num_kv_heads,
               num_seqs,     num_q_heads, head_dim,     block_size,   max_blocks_per_seq,
               num_blocks,   workspace,   workspace_bytes, (cudaStream_t)stream};
  if (dtype == PA_BF16) return dispatch_shape<__nv_bfloat16>(a, dev, sms);
  return dispatch_shape<__half>(a, dev, sms);
}

int pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping, int num_pairs,
                   int num_kv_heads, int head_dim, int block_size, int num_blocks,
                   pa_dtype dtype, pa_stream_t stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks < 0)
    return PA_ERR_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_ARG;
  if (!supported_shape(head_dim, block_size)) return PA_ERR_UNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  if (num_pairs > 65535) return PA_ERR_UNSUPPORTED;
  if (!k_cache || !v_cache || !block_mapping) return PA_ERR_ARG;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(block_mapping, 8))
    return PA_ERR_ARG;
  const long long vec_per_block = (long long)num_kv_heads * block_size * head_dim * 2 / 16;
  const unsigned chunks = (unsigned)((vec_per_block + pa::kCopyPerCta - 1) / pa::kCopyPerCta);
  dim3 grid(chunks, (unsigned)num_pairs);
  pa::copy_blocks_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(
      static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), block_mapping, vec_per_block,
      num_blocks);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_device_error(unsigned *flags, int clear) {
  if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, pa::g_device_error, sizeof(v)) != cudaSuccess) return PA_ERR_CUDA;
  if (clear && v) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(pa::g_device_error, &zero, sizeof(zero)) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  if (flags) *flags = v;
  return v ? PA_ERR_DEVICE_BOUNDS : PA_OK;
}

int pa_paged_decode_attention_no_alloc(float *out, const void *q, const void *k_cache,
                                       const void *v_cache, const int32_t *block_tables,
                                       const int32_t *context_lens, float scale,
                                       int num_kv_heads, int num_seqs, int num_q_heads,
                                       int head_dim, int block_size, int max_blocks_per_seq,
                                       int max_context_len, int num_blocks, pa_dtype dtype,
                                       pa_stream_t stream) {
  if (num_seqs < 0 || num_kv_heads <= 0 || num_q_heads <= 0 || head_dim <= 0 || block_size <= 0)
    return PA_ERR_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_ARG;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_ARG;
  if (!supported_shape(head_dim, block_size) || num_q_heads / num_kv_heads > 16)
    return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (max_blocks_per_seq <= 0 || num_blocks <= 0 || max_context_len < 0 ||
      (long long)max_context_len > (long long)max_blocks_per_seq * block_size)
    return PA_ERR_ARG;
  if ((long long)num_blocks * num_kv_heads * block_size >= (1ll << 31)) return PA_ERR_UNSUPPORTED;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PA_ERR_ARG;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return PA_ERR_ARG;
  int dev;
  if (current_device(&dev) != PA_OK || dev >= kMaxDevices) return PA_ERR_CUDA;
  const int sms = sm_count(dev);
  if (sms <= 0) return PA_ERR_CUDA;
  void *scratch = nullptr;
  const int st = no_alloc_scratch(dev, &scratch);
  if (st != PA_OK) return st;
  // The scratch needs no clearing: every partial the merge reads is written
  // by the same call's streaming kernel first.  A launch that needs more than
  // kNoAllocScratchBytes is refused by launch_decode with PA_ERR_WORKSPACE.
  DecodeArgs a{out,          q,           k_cache,      v_cache,      nullptr,
               nullptr,      block_tables, context_lens, scale,        num_kv_heads,
               num_seqs,     num_q_heads, head_dim,     block_size,   max_blocks_per_seq,
               num_blocks,   scratch,     kNoAllocScratchBytes, (cudaStream_t)stream};
  if (dtype == PA_BF16) return dispatch_shape<__nv_bfloat16>(a, dev, sms);
  return dispatch_shape<__half>(a, dev, sms);
}

int pa_paged_prefill_attention(float *out, const void *q, const void *k_cache,
                               const void *v_cache, const int32_t *block_tables,
                               const int32_t *context_lens, const int32_t *query_start,
                               float scale, int num_kv_heads, int num_seqs, int num_tokens,
                               int num_q_heads, int head_dim, int block_size,
                               int max_blocks_per_seq, int max_query_len, int num_blocks,
                               pa_dtype dtype, pa_stream_t stream) {
  if (num_seqs < 0 || num_tokens < 0 || max_query_len < 0 || num_kv_heads <= 0 ||
      num_q_heads <= 0 || head_dim <= 0 || block_size <= 0)
    return PA_ERR_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_ARG;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_ARG;
  if (!supported_shape(head_dim, block_size) || num_q_heads / num_kv_heads > 16)
    return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0 || num_tokens == 0 || max_query_len == 0) return PA_OK;
  if (max_blocks_per_seq <= 0 || num_blocks <= 0) return PA_ERR_ARG;
  if ((long long)num_blocks * num_kv_heads * block_size >= (1ll << 31)) return PA_ERR_UNSUPPORTED;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start)
    return PA_ERR_ARG;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(query_start, 4))
    return PA_ERR_ARG;
  int dev;
  if (current_device(&dev) != PA_OK || dev >= kMaxDevices) return PA_ERR_CUDA;
  PrefillArgs a{out,          q,           k_cache,       v_cache,     block_tables,
                context_lens, query_start, scale,         num_kv_heads, num_seqs,
                num_tokens,   num_q_heads, head_dim,      block_size,  max_blocks_per_seq,
                max_query_len, num_blocks, (cudaStream_t)stream};
  if (dtype == PA_BF16) return dispatch_prefill<__nv_bfloat16>(a, dev);
  return dispatch_prefill<__half>(a, dev);
}

int pa_set_wait_limit(long long ns) {
  if (ns < 0) return PA_ERR_ARG;
  g_wait_limit_ns.store(ns == 0 ? kDefaultWaitLimitNs : (unsigned long long)ns);
  return PA_OK;
}

int pa_decode_tuning(int nstage, int ctas_per_sm, int min_tiles_per_warp) {
  if (nstage < 0 || ctas_per_sm < 0 || ctas_per_sm > kMaxCtasPerSm || min_tiles_per_warp < 0)
    return PA_ERR_ARG;
  g_tune_nstage.store(nstage);
  g_tune_ctas.store(ctas_per_sm);
  g_tune_min_tiles.store(min_tiles_per_warp);
  return PA_OK;
}

}  // extern "C"
