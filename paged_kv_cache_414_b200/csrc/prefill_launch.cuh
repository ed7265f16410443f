// Host side of chunked-prefill attention: tensor maps and the launch.
// Included by pa_kernels.cu inside its anonymous namespace (which provides
// encode_fn, encode_pool_map, kMaxDevices and g_wait_limit_ns); kept apart so
// that the decode kernels' launch code can be identified on its own.
#pragma once

// Q [T, Hq, D] as a 3-D map (D, Hq, T); a box is 64 columns x the G heads of
// one kv head x TQ tokens, i.e. 128 query rows ordered (token, head).
bool encode_query_map(CUtensorMap *m, const void *q, int T, int Hq, int D, int G, int tq) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
  cuuint32_t box[3] = {64u, (cuuint32_t)G, (cuuint32_t)tq};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void *>(q), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// out [T, Hq, D] fp32 as a 3-D map (D, Hq, T) for the prefill epilogue's TMA
// stores: a box is 32 columns x the G heads of one kv head x TQ tokens,
// 128-byte swizzled in shared memory.
bool encode_out_map(CUtensorMap *m, float *out, int T, int Hq, int D, int G, int tq) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)Hq * D * 4};
  cuuint32_t box[3] = {32u, (cuuint32_t)G, (cuuint32_t)tq};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, out, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct PrefillArgs {
  float *out;
  const void *q, *k_cache, *v_cache;
  const int32_t *block_tables, *context_lens, *query_start;
  float scale;
  int num_kv_heads, num_seqs, num_tokens, num_q_heads, head_dim, block_size, max_blocks,
      max_query_len, num_blocks;
  cudaStream_t stream;
};

template <typename T, int D, int B>
int launch_prefill(const PrefillArgs &a, int dev) {
  using L = pa::PrefillSmem<D>;
  auto kern = pa::paged_prefill_kernel<T, D, B>;
  static std::atomic<int> attr_set[kMaxDevices];
  if (!attr_set[dev].load()) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES) !=
        cudaSuccess)
      return PA_ERR_CUDA;
    attr_set[dev].store(1);
  }
  const int G = a.num_q_heads / a.num_kv_heads;
  const int tq = pa::kPfRows / G;
  CUtensorMap qmap, kmap, vmap, omap;
  const long long rows = (long long)a.num_blocks * a.num_kv_heads * B;
  if (!encode_query_map(&qmap, a.q, a.num_tokens, a.num_q_heads, D, G, tq) ||
      !encode_pool_map(&kmap, a.k_cache, rows, D, B) ||
      !encode_pool_map(&vmap, a.v_cache, rows, D, B) ||
      !encode_out_map(&omap, a.out, a.num_tokens, a.num_q_heads, D, G, tq))
    return PA_ERR_CUDA;
  pa::PrefillParams p;
  p.out = a.out;
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  p.query_start = a.query_start;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.num_seqs = a.num_seqs;
  p.num_tokens = a.num_tokens;
  p.num_q_heads = a.num_q_heads;
  p.num_kv_heads = a.num_kv_heads;
  p.group = G;
  p.max_blocks = a.max_blocks;
  p.num_blocks = a.num_blocks;
  p.tq = tq;
  p.q_tiles = (a.max_query_len + 2 * tq - 1) / (2 * tq);   // a CTA takes two query tiles
  p.wait_ns = g_wait_limit_ns.load();
  const long long nx = (long long)p.q_tiles * a.num_seqs * a.num_kv_heads;
  if (nx >= (1ll << 31)) return PA_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nx);   // (sequence by rank, query-tile pair, kv head)
  cfg.blockDim = dim3(pa::kPfThreads);
  cfg.dynamicSmemBytes = L::BYTES;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, qmap, kmap, vmap, omap, p) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

template <typename T>
int dispatch_prefill(const PrefillArgs &a, int dev) {
  if (a.head_dim == 128 && a.block_size == 16) return launch_prefill<T, 128, 16>(a, dev);
  if (a.head_dim == 128 && a.block_size == 32) return launch_prefill<T, 128, 32>(a, dev);
  if (a.head_dim == 64 && a.block_size == 16) return launch_prefill<T, 64, 16>(a, dev);
  return launch_prefill<T, 64, 32>(a, dev);
}

