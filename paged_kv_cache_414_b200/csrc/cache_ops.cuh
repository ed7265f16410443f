// Cache write (reshape_and_cache) and copy-on-write block copy (copy_blocks).
//
// reshape_and_cache: "Why OS Virtual Memory Paging Saved LLM Inference: The
// vLLM Breakthrough", section 2, on-demand allocation -- each new token's K/V
// is written into the slot its sequence's block table assigns.
// copy_blocks: same page, section 3 "Copy-on-Write for Prompt Sharing" -- a
// branch that writes into a shared block gets a private copy of it.
//
// Both are pure 16-byte-vector copies; both are HBM-bound with one read and
// one write of every byte moved.
#pragma once

#include <stdint.h>

#include "pa_device.cuh"

namespace pa {

// One thread per 16-byte vector of one (token, kv head) row, for K and V.
// key/value rows are [num_tokens, Hkv, D]; the pool is [NB, Hkv, B, D].
__global__ void __launch_bounds__(256)
    reshape_and_cache_kernel(const uint4 *__restrict__ key, const uint4 *__restrict__ value,
                             uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                             const int64_t *__restrict__ slot_mapping, long long num_vec,
                             int vec_per_row, int num_kv_heads, int block_size,
                             long long num_slots) {
  allow_dependent_launch();   // the decode kernel may get scheduled meanwhile
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < num_vec; i += stride) {
    const long long row = i / vec_per_row;          // token * Hkv + head
    const int c = (int)(i - row * vec_per_row);
    const long long t = row / num_kv_heads;
    const int h = (int)(row - t * num_kv_heads);
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (c == 0 && h == 0) flag_error(PA_DEVERR_SLOT);
      continue;
    }
    const long long blk = slot / block_size;
    const int off = (int)(slot - blk * block_size);
    const long long dst = ((blk * num_kv_heads + h) * block_size + off) * vec_per_row + c;
    k_cache[dst] = __ldg(key + i);
    v_cache[dst] = __ldg(value + i);
  }
}

// Grid (chunks, pairs): block (x, pair) copies vectors [x * kCopyPerCta,
// (x + 1) * kCopyPerCta) of the pair's block, in both pools.  Each thread
// loads all its vectors before it stores any: the caller guarantees that no
// destination block is also a source, so the loads never see this kernel's
// stores, and a thread keeps 2 * kCopyUnroll 16-byte loads in flight.
constexpr int kCopyUnroll = 4;
constexpr int kCopyPerCta = 256 * kCopyUnroll;
__global__ void __launch_bounds__(256)
    copy_blocks_kernel(uint4 *k_cache, uint4 *v_cache, const int64_t *__restrict__ block_mapping,
                       long long vec_per_block, int num_blocks) {
  allow_dependent_launch();
  const long long pair = blockIdx.y;
  const int64_t src = __ldg(block_mapping + 2 * pair);
  const int64_t dst = __ldg(block_mapping + 2 * pair + 1);
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(PA_DEVERR_COPY_PAIR);
    return;
  }
  const long long beg = (long long)blockIdx.x * kCopyPerCta + threadIdx.x;
  const uint4 *ks = k_cache + src * vec_per_block;
  const uint4 *vs = v_cache + src * vec_per_block;
  uint4 *kd = k_cache + dst * vec_per_block;
  uint4 *vd = v_cache + dst * vec_per_block;
  uint4 kr[kCopyUnroll], vr[kCopyUnroll];
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const long long i = beg + u * 256;
    if (i < vec_per_block) {
      kr[u] = ks[i];
      vr[u] = vs[i];
    }
  }
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const long long i = beg + u * 256;
    if (i < vec_per_block) {
      kd[i] = kr[u];
      vd[i] = vr[u];
    }
  }
}

}  // namespace pa
