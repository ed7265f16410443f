// Chunked-prefill attention over the paged KV cache, on the fifth-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// What it computes ("Can OS paging techniques reduce LLM serving memory
// waste?", second paragraph: attention runs block by block over blocks that
// need not be contiguous; "Why OS Virtual Memory Paging Saved LLM Inference:
// The vLLM Breakthrough", section 2: the KV cache fills as tokens arrive, the
// block table maps logical to physical blocks).  Sequence s adds a chunk of
// C_s tokens whose K/V are already in the cache; its context holds
// L_s >= C_s tokens.  Chunk token i sits at position L_s - C_s + i and attends
// causally to positions 0 .. L_s - C_s + i:
//   out[t, h] = softmax(scale * q[t, h] . K_s[0..p]) V_s[0..p].
//
// Work split: one CTA per (sequence, kv head, pair of query tiles), launched
// longest sequence first (ranked in the kernel for up to 32 sequences).  A query
// tile is 128 rows = TQ = 128 / G chunk tokens x the G query heads that share
// the kv head; the CTA's two tiles (A, then B: 2 TQ consecutive tokens) share
// every K/V tile fetched from the pool.  Keys go in tiles of 128 positions
// (8 blocks of 16 or 4 of 32), fetched by TMA straight from their physical
// blocks into 128-byte-swizzled shared memory.
//
//   warp 0      TMA producer: both Q tiles once, then K/V tiles into a ring;
//               each lane issues one copy of a tile (one block, one 64-column
//               chunk, K or V), and K and V land on separate barriers; K and V
//               of a stage are released separately.
//   warp 1      owns the tensor memory and issues the MMAs (the whole warp
//               runs the loop, one elected lane issues), alternating
//               between the query tiles so that one tile's MMAs run while the
//               other tile's softmax does:
//                 S_X = Q_X K_j^T   (M 128, N 128 keys, K = head_dim, cache dtype)
//                 O_X += P_X V_j    (M 128, N = head_dim, K 128 keys, fp16)
//               in the order S_A(0) S_B(0), then per tile j: O_A += P_A V_j,
//               S_A(j+1), O_B += P_B V_j, S_B(j+1).
//   warps 2-9   softmax of tile A, warps 10-17 of tile B, two threads per
//               row: warps w and w+4 share the tensor-memory lanes of one row
//               quarter and take 64 keys each, exchanging partial maxima every
//               tile (through shared memory, ordered by a 64-arrival mbarrier
//               per pair and the same bounded wait as everything else) and
//               partial sums once at the end.  Online maximum and sum in
//               fp32; the weights go to tensor memory as fp16 (the row sums
//               add the rounded values, so the normalisation matches what the
//               MMA multiplies), where the P.V MMA reads them as its A operand.
//               O is rescaled in tensor memory when the row maximum moves by
//               more than 2^8; the epilogue writes out = O / l, full query
//               tiles through shared memory and TMA stores.
//   warps 18-23 V converter: zero the rows of a V tile past the last visible
//               key and, for bf16 caches, rewrite the tile in place as fp16
//               (exact for |v| <= 65504; a value beyond fp16's range becomes
//               infinite, the outputs it reaches come out non-finite, and the
//               epilogue reports PA_DEVERR_RANGE), so P.V is one fp16 MMA per
//               16 keys.  The conversion sits between a V tile's arrival and
//               its P.V, so it gets six warps (at 768 threads every thread
//               keeps 80 registers: the softmax re-reads its scores from TMEM
//               rather than holding them).
//
// Tensor memory (512 columns): tile A's S at 0 and O at 128, tile B's S at
// 256 and O at 384.  P replaces S in its own columns: each key half's 64
// fp16 weights (two per column) fill the first 32 of its 64 score columns.
// The MMA that next writes a tile's S columns is issued after that tile's
// P.V, and MMAs run in issue order.
//
// Every wait is bounded: on time-out a shared abort flag stops every role,
// PA_DEVERR_TIMEOUT is set, copies and MMAs in flight are waited for (again
// bounded) and the tensor memory is freed.
#pragma once

#include <limits.h>
#include <math.h>

#include <type_traits>

#include "umma.cuh"

namespace pa {

struct PrefillParams {
  float *out;                    // [T, Hq, D]
  const int32_t *block_tables;   // [S, max_blocks]
  const int32_t *context_lens;   // [S]
  const int32_t *query_start;    // [S + 1]
  float scale_log2;              // scale * log2(e)
  int num_seqs, num_tokens, num_q_heads, num_kv_heads, group, max_blocks, num_blocks;
  int q_tiles;                   // CTAs (pairs of query tiles) per sequence in the grid
  int tq;                        // chunk tokens per query tile (128 / group)
  uint64_t wait_ns;              // limit of a wait before giving up (2 s by default)
};

constexpr int kPfRows = 128;      // query rows per query tile
constexpr int kPfKeys = 128;      // keys per K/V tile
constexpr int kPfThreads = 768;   // producer, MMA, 2 x 8 softmax warps, 6 V-converter warps
constexpr int kPfConv = 192;      // V-converter threads
constexpr uint32_t kPfTmemCols = 512;
constexpr uint64_t kPfDrainLimitNs = 2000000000ull;   // draining after an abort

template <int D>
struct PrefillSmem {
  static constexpr int NCH = D / 64;                  // 64-column chunks of a row
  static constexpr int STAGES = D == 128 ? 2 : 3;     // K/V ring depth
  static constexpr int REGION = kPfRows * 128;        // one 64-column chunk of 128 rows
  static constexpr int Q_TILE = NCH * REGION;         // one query tile
  static constexpr int KV_BYTES = NCH * kPfKeys * 128;
  static constexpr int OFF_Q = 0;                     // two query tiles
  static constexpr int OFF_K = OFF_Q + 2 * Q_TILE;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * KV_BYTES;
  static constexpr int OFF_X = OFF_BAR + 512;         // pair exchange: [tile][set][half][row]
  static constexpr int BYTES = OFF_X + 2 * 3 * 2 * 128 * 4 + 1024;  // + alignment slack
};

// Bounded wait that also gives up when another role has aborted.
__device__ __forceinline__ bool pf_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                        uint64_t limit_ns) {
  bool done;
  if (limit_ns < kShortWaitNs) {            // a short limit set on purpose: poll, count cycles
    const long long c0 = clock64();
    while (!(done = mbar_test_wait(bar, parity)) && !*abort &&
           (uint64_t)(clock64() - c0) <= 2 * limit_ns) {
    }
  } else {
    done = mbar_try_wait(bar, parity);
    const uint64_t t0 = done ? 0 : globaltimer_ns();
    while (!done && !*abort && globaltimer_ns() - t0 <= limit_ns) done = mbar_try_wait(bar, parity);
  }
  if (done) return true;
  if (!*abort) {
    *abort = 1;
    flag_error(PA_DEVERR_TIMEOUT);
  }
  return false;
}

// 2^x by the hardware approximation (ex2.approx, flush-to-zero); its error is
// far below the rounding the weights then get.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Packed pairs of fp32 lanes (one instruction for two values): (a0, a1) * b + c
// and a + b on the pairs.
__device__ __forceinline__ void ffma2(float &d0, float &d1, float a0, float a1, float b0,
                                      float b1, float c0, float c1) {
  asm("{\n\t.reg .b64 a, b, c, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\tmov.b64 c, {%6, %7};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void fadd2(float &d0, float &d1, float a0, float a1, float b0,
                                      float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void fsub2(float &d0, float &d1, float a0, float a1, float b0,
                                      float b1) {
  asm("{\n\t.reg .b64 a, b, d;\n\t"
      "mov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "sub.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// A packed pair of bf16 values as a packed pair of fp16 values: exact within
// fp16's range (bf16 has fewer significant bits); a value beyond it
// (|v| >= 65520) becomes infinite.  No range test here: an infinite V makes
// every output row of the tile that reads it non-finite, which the epilogue
// checks once per row instead of once per element.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t x) {
  const float hi = __uint_as_float(x & 0xffff0000u), lo = __uint_as_float(x << 16);
  uint32_t y;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(y) : "f"(hi), "f"(lo));
  return y;
}

// Two weights rounded to fp16 (packed, the first in the low half); the
// rounded values are what the row sums add, so the normalisation matches
// what the MMA multiplies.
__device__ __forceinline__ uint32_t round_f16(float a, float b, float *s0, float *s1) {
  __half2 h = __floats2half2_rn(a, b);
  const float2 f = __half22float2(h);
  fadd2(*s0, *s1, *s0, *s1, f.x, f.y);
  return *reinterpret_cast<uint32_t *>(&h);
}

template <typename T, int D, int B>
__global__ void __launch_bounds__(kPfThreads, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap qmap,
                         const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap,
                         const __grid_constant__ CUtensorMap omap, const PrefillParams p) {
  using L = PrefillSmem<D>;
  constexpr int NCH = L::NCH;
  constexpr int NST = L::STAGES;
  constexpr int BPT = kPfKeys / B;                    // blocks per K/V tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem + L::OFF_Q;
  uint8_t *sK = smem + L::OFF_K;
  uint8_t *sV = smem + L::OFF_V;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::OFF_BAR);
  uint64_t *full_k = bars + 0;     // [NST] K tile landed
  uint64_t *full_v = bars + 3;     // [NST] V tile landed
  uint64_t *empty_k = bars + 6;    // [NST] K tile consumed by both query tiles' S
  uint64_t *empty_v = bars + 27;   // [NST] V tile consumed by both query tiles' P.V
  uint64_t *q_full = bars + 9;     // both Q tiles landed
  uint64_t *s_full = bars + 10;    // [query tile] S written
  uint64_t *p_full = bars + 12;    // [query tile] P written, O rescaled (256 arrivals)
  uint64_t *o_done = bars + 14;    // [query tile] O += P V done
  uint64_t *drain = bars + 16;     // every MMA done (before freeing tensor memory)
  uint64_t *pair = bars + 17;      // [query tile][row quarter] the two threads of a row
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 25);
  volatile int *abort = reinterpret_cast<volatile int *>(bars + 26);
  uint64_t *v_ready = bars + 32;   // [NST] V tile in fp16 with its tail zeroed

  float *xch = reinterpret_cast<float *>(smem + L::OFF_X);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.group;

  grid_dependency_wait();     // the chunk's cache write may be the kernel before
  // Work unit of this CTA: (sequence, pair of query tiles, kv head), the kv
  // head varying fastest in launch order.  A unit's length is set by its
  // sequence's context, so with up to 32 sequences they are ranked by
  // context length (longest first, ties by index) and the launch order runs
  // through them by rank: the longest units start first and the short ones
  // fill the last wave.  More sequences keep the plain order (query-tile
  // pair slowest), which balances about as well.
  const int kh = blockIdx.x % p.num_kv_heads;
  const int v = blockIdx.x / p.num_kv_heads;
  int s, qt;
  if (p.num_seqs <= 32) {
    __shared__ int seq_of_rank;
    const int rank_wanted = v / p.q_tiles;
    qt = p.q_tiles - 1 - v % p.q_tiles;
    if (warp == 0) {
      const int Lm = lane < p.num_seqs ? __ldg(p.context_lens + lane) : INT_MIN;
      int rank = 0;
      for (int k = 0; k < p.num_seqs; ++k) {
        const int Lk = __shfl_sync(0xffffffffu, Lm, k);
        rank += (Lk > Lm || (Lk == Lm && k < lane)) ? 1 : 0;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, lane < p.num_seqs && rank == rank_wanted);
      if (lane == 0) seq_of_rank = __ffs(hit) - 1;
    }
    __syncthreads();
    s = seq_of_rank;
  } else {
    s = v % p.num_seqs;
    qt = p.q_tiles - 1 - v / p.num_seqs;
  }
  const int q0 = __ldg(p.query_start + s);
  const int C = __ldg(p.query_start + s + 1) - q0;
  const int Lc = __ldg(p.context_lens + s);
  const int tok0 = qt * 2 * p.tq;
  if (C < 0 || C > Lc || Lc > p.max_blocks * B || q0 < 0 || q0 + C > p.num_tokens) {
    if (threadIdx.x == 0 && kh == 0 && qt == 0) flag_error(PA_DEVERR_CONTEXT_LEN);
    return;
  }
  // a chunk longer than the grid covers (max_query_len too small): its last
  // rows are not computed; say so
  if (threadIdx.x == 0 && kh == 0 && qt == 0 && C > p.q_tiles * 2 * p.tq)
    flag_error(PA_DEVERR_CONTEXT_LEN);
  if (tok0 >= C) return;                               // uniform over the CTA
  const int ntok = min(2 * p.tq, C - tok0);
  const int pos_max = Lc - C + tok0 + ntok - 1;        // last position any row sees
  const int n_tiles = pos_max / kPfKeys + 1;
  const int nb_used = pos_max / B + 1;                 // blocks holding positions 0..pos_max
  const int rows_q = p.tq * G;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full_k[i], 1);
      mbar_init(&full_v[i], 1);
      mbar_init(&empty_k[i], 1);
      mbar_init(&empty_v[i], 1);
      mbar_init(&v_ready[i], kPfConv);
    }

    mbar_init(q_full, 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 256);
      for (int q = 0; q < 4; ++q) mbar_init(&pair[x * 4 + q], 64);
      mbar_init(&o_done[x], 1);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kPfTmemCols);
    tmem_relinquish();
  }
  if (rows_q < kPfRows) {     // Q rows no chunk token fills: zeros, not stale bits
    const int per_tile = NCH * (kPfRows - rows_q) * 8;
    for (int i = threadIdx.x; i < 2 * per_tile; i += kPfThreads) {
      const int x = i / per_tile, rem0 = i % per_tile;
      const int c = rem0 / ((kPfRows - rows_q) * 8), rem = rem0 % ((kPfRows - rows_q) * 8);
      *reinterpret_cast<uint4 *>(sQ + x * L::Q_TILE + c * L::REGION + (rows_q + rem / 8) * 128 +
                                 (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // lane -> (block of the tile, 64-column chunk, K or V): BPT * NCH * 2 <= 32 copies
    constexpr int NCOPY = BPT * NCH * 2;
    const int cb = lane / (NCH * 2), cc = (lane >> 1) % NCH, ckv = lane & 1;
    if (lane == 0) {
      prefetch_tensormap(&qmap);
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
      // tile B past the chunk: load tile A's tokens again (finite, never stored)
      const int zb = tok0 + p.tq < C ? q0 + tok0 + p.tq : q0 + tok0;
      mbar_arrive_expect_tx(q_full, 2 * NCH * 128 * rows_q);
      for (int c = 0; c < NCH; ++c) {
        tma_load_3d(sQ + c * L::REGION, &qmap, c * 64, kh * G, q0 + tok0, q_full);
        tma_load_3d(sQ + L::Q_TILE + c * L::REGION, &qmap, c * 64, kh * G, zb, q_full);
      }
    }
    const int32_t *table = p.block_tables + (size_t)s * p.max_blocks;
    // K and V of a stage are released separately: K as soon as both query
    // tiles' S of its tile ran, V after their P.V, so the next K load starts
    // about one tile earlier than a joint release would allow.
    int issued_k = 0, issued_v = 0;
    for (int j = 0; j < n_tiles; ++j) {
      const int st = j % NST;
      // this lane's block id, fetched before the stage is free
      const int b0 = j * BPT;
      int id = -1;
      bool bad = false;
      if (lane < NCOPY && cb < nb_used - b0) {
        const int v = __ldg(table + b0 + cb);
        if (v >= 0 && v < p.num_blocks) id = v; else bad = true;
      }
      if (bad && cc == 0 && ckv == 0) flag_error(PA_DEVERR_BLOCK_ID);
      const unsigned valid = __ballot_sync(0xffffffffu, id >= 0);
      const int off = st * L::KV_BYTES + cc * kPfKeys * 128 + cb * B * 128;
      const int row = (id * p.num_kv_heads + kh) * B;
      if (j >= NST) {
        const bool w =
            lane == 0 ? pf_wait(&empty_k[st], (j / NST - 1) & 1, abort, p.wait_ns) : true;
        if (!__shfl_sync(0xffffffffu, w, 0)) break;
      }
      if (lane == 0) mbar_arrive_expect_tx(&full_k[st], __popc(valid & 0x55555555u) * B * 128);
      __syncwarp();
      if (id >= 0 && ckv == 0) tma_load_2d(sK + off, &kmap, cc * 64, row, &full_k[st]);
      issued_k = j + 1;
      if (j >= NST) {
        const bool w =
            lane == 0 ? pf_wait(&empty_v[st], (j / NST - 1) & 1, abort, p.wait_ns) : true;
        if (!__shfl_sync(0xffffffffu, w, 0)) break;
      }
      if (lane == 0) mbar_arrive_expect_tx(&full_v[st], __popc(valid & 0xAAAAAAAAu) * B * 128);
      __syncwarp();
      if (id >= 0 && ckv == 1) tma_load_2d(sV + off, &vmap, cc * 64, row, &full_v[st]);
      issued_v = j + 1;
    }
    // copies still in flight must land before the CTA exits
    if (lane == 0) {
      for (int j = max(0, issued_k - NST); j < issued_k; ++j)
        mbar_wait_bounded(&full_k[j % NST], (j / NST) & 1, kPfDrainLimitNs);
      for (int j = max(0, issued_v - NST); j < issued_v; ++j)
        mbar_wait_bounded(&full_v[j % NST], (j / NST) & 1, kPfDrainLimitNs);
      mbar_wait_bounded(q_full, 0, kPfDrainLimitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    // (whole warp, warp-uniform waits; the wrappers elect the issuing lane)
    {
      constexpr bool kBf = std::is_same<T, __nv_bfloat16>::value;
      const uint32_t idS = umma_idesc_f16(kBf, kPfRows, kPfKeys, false, false);
      const uint32_t idO16 = umma_idesc_f16(false, kPfRows, D, false, true);   // fp16 P and V
      const uint32_t aQ = smem_addr(sQ), aK = smem_addr(sK), aV = smem_addr(sV);
      // Shared-memory descriptors, built once: a k-step moves the start
      // address field by a constant, so every MMA below takes a
      // precomputed base plus an immediate (the issuing warp shares its
      // scheduler with softmax warps, so its instruction count per MMA is
      // what sets the issue rate).
      const uint64_t dQ0 = umma_desc_sw128(aQ, 16, 1024);
      const uint64_t dK0 = umma_desc_sw128(aK, 16, 1024);
      const uint64_t dV0 = umma_desc_sw128(aV, kPfKeys * 128, 1024);
      constexpr uint32_t kStageStep = L::KV_BYTES >> 4, kQStep = L::Q_TILE >> 4;
      auto issue_s = [&](int x, int j) {        // S_x = Q_x K_j^T
        const uint64_t dq = dQ0 + x * kQStep, dk = dK0 + (j % NST) * kStageStep;
        const uint32_t d = tmem + x * 256;
        constexpr uint32_t kRegion = L::REGION >> 4;
        if constexpr (D == 128)
          umma_ss_group8<0, 2, 4, 6, kRegion, kRegion + 2, kRegion + 4, kRegion + 6>(d, dq, dk,
                                                                                      idS, 0u);
        else
          umma_ss_group4<0, 2, 4, 6>(d, dq, dk, idS, 0u);
        umma_commit(&s_full[x]);
      };
      auto issue_pv = [&](int x, int j) {       // O_x += P_x V_j, fp16 P and V
        const uint64_t dv = dV0 + (j % NST) * kStageStep;
        const uint32_t pj = tmem + x * 256, d = pj + 128;
        const uint32_t acc0 = j > 0 ? 1u : 0u;
        // 16 keys per step: 8 columns of P, 16 rows of V
        umma_ts_group8<0, 8, 16, 24, 64, 72, 80, 88, 0, 128, 256, 384, 512, 640, 768, 896>(
            d, pj, dv, idO16, acc0);
        umma_commit(&o_done[x]);
      };
      // every lane waits; the warp goes on only if all of them saw the phase
      auto wait_all = [&](uint64_t *bar, uint32_t parity) {
        return __all_sync(0xffffffffu, pf_wait(bar, parity, abort, p.wait_ns));
      };
      bool ok = wait_all(q_full, 0) && wait_all(&full_k[0], 0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        umma_commit(&empty_k[0]);
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        // tile A: its P.V, then its next S (which overwrites its P, in issue order)
        if (!wait_all(&p_full[0], j & 1)) break;
        if (!wait_all(&v_ready[j % NST], (j / NST) & 1)) break;
        tc_fence_after();
        issue_pv(0, j);
        const bool more = j + 1 < n_tiles;
        if (more) {
          if (!wait_all(&full_k[(j + 1) % NST], ((j + 1) / NST) & 1)) break;
          tc_fence_after();
          issue_s(0, j + 1);
        }
        // tile B
        if (!wait_all(&p_full[1], j & 1)) break;
        tc_fence_after();
        issue_pv(1, j);
        umma_commit(&empty_v[j % NST]);
        if (more) {
          issue_s(1, j + 1);
          umma_commit(&empty_k[(j + 1) % NST]);
        }
      }
      umma_commit(drain);
      mbar_wait_bounded(drain, 0, kPfDrainLimitNs);
    }
  } else if (warp >= 18) {
    // ------------------------------------------------------------ V converter
    // Each landed V tile, before its P.V: rows past the last visible key are
    // zeroed (masked for every row, but 0 x NaN from stale or poisoned bits
    // would reach O), and a bf16 tile is rewritten in place as fp16 -- exact
    // for |v| <= 65504, fp16's largest value; beyond it the value becomes
    // infinite and the epilogue reports the non-finite rows -- so that P.V
    // takes one fp16 P.  An element keeps its byte position, so the swizzle
    // is untouched.  The conversion's instruction count matters: these warps
    // share their schedulers with the softmax.
    const int ct = threadIdx.x - 18 * 32;          // 0 .. kPfConv - 1
    constexpr int NCHUNK = NCH * kPfKeys * 8;      // 16-byte chunks of a V tile
    constexpr bool kBf = std::is_same<T, __nv_bfloat16>::value;
    for (int j = 0; j < n_tiles; ++j) {
      const int st = j % NST;
      if (!__all_sync(0xffffffffu, pf_wait(&full_v[st], (j / NST) & 1, abort, p.wait_ns)))
        break;
      uint8_t *v0 = sV + st * L::KV_BYTES;
      const int z0 = j == n_tiles - 1 ? pos_max + 1 - j * kPfKeys : kPfKeys;   // first dead row
      for (int i = ct; i < NCHUNK; i += kPfConv) {
        uint4 *c = reinterpret_cast<uint4 *>(v0 + i * 16);
        if (((i >> 3) & (kPfKeys - 1)) >= z0) {
          *c = make_uint4(0, 0, 0, 0);
        } else if (kBf) {
          const uint4 w = *c;
          *c = make_uint4(bf16x2_to_f16x2(w.x), bf16x2_to_f16x2(w.y), bf16x2_to_f16x2(w.z),
                          bf16x2_to_f16x2(w.w));
        }
      }
      // generic-proxy writes, read next by the tensor cores (async proxy)
      fence_proxy_async_smem();
      mbar_arrive(&v_ready[st]);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int x = (warp - 2) >> 3;                // query tile: warps 2-9 A, 10-17 B
    const int half = ((warp - 2) >> 2) & 1;       // keys 64*half .. 64*half+63 of a tile
    const int quarter = warp & 3;                 // tensor-memory lanes 32*quarter ..
    const int r = quarter * 32 + lane;            // this thread's row of the tile
    const int t = r / G, g = r - (r / G) * G;
    const int tokx = tok0 + x * p.tq;             // the tile's first chunk token
    const bool row_ok = r < rows_q && tokx + t < C;
    const int pos = row_ok ? Lc - C + tokx + t : pos_max;
    const int pos_min = min(Lc - C + tokx, pos_max);
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const uint32_t tSx = tmem + x * 256 + lane_addr, tOx = tSx + 128;
    uint64_t *pr_bar = &pair[x * 4 + quarter];
    // exchange slots: [tile][set: tile parity 0/1, 2 = row sums][half][row]
    auto slot = [&](int set, int hf) { return xch + ((x * 3 + set) * 2 + hf) * 128 + r; };
    const float sl2 = p.scale_log2;
    const bool pos_scale = sl2 > 0.f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      ok = __all_sync(0xffffffffu, pf_wait(&s_full[x], j & 1, abort, p.wait_ns));
      if (!ok) break;
      tc_fence_after();
      // this half's 64 scores: read for the maximum, then read again 32 at a
      // time for the weights (keeping all 64 in registers costs spills)
      const uint32_t sj = tSx + half * 64;
      const int kh0 = j * kPfKeys + half * 64;   // first key of this half
      const bool diag = kh0 + 63 > pos_min;      // some key past some row's position
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t v[32];
        tmem_load32(sj + hh * 32, v);
        if (!pos_scale) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (kh0 + hh * 32 + i <= pos) mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(v[i]) * sl2);
        } else if (diag) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (kh0 + hh * 32 + i <= pos) mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(v[i]));
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            mx[i & 7] = fmax3(mx[i & 7], __uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
        }
      }
      float mr = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                       fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      // the row's maximum: exchange with the other half (two slot sets by tile
      // parity, so a partner still reading this tile's value is never
      // overwritten by the next tile's)
      *slot(j & 1, half) = mr;
      mbar_arrive(pr_bar);
      ok = __all_sync(0xffffffffu, pf_wait(pr_bar, j & 1, abort, p.wait_ns));
      if (!ok) break;
      mr = fmaxf(mr, *reinterpret_cast<volatile float *>(slot(j & 1, 1 - half)));
      // with a positive scale the maximum of the raw scores, scaled once
      const float mt = pos_scale ? mr * sl2 : mr;
      // Lazy rescaling: the reference maximum m moves only when the tile's
      // maximum exceeds it by more than 8 (log2 units), so weights stay below
      // 2^8 and O is rescaled in tensor memory only on those rare steps.  Both
      // halves of a row take the same decisions.
      const bool bump = mt > m + 8.f;
      const float m_new = bump ? mt : m;
      const float alpha = bump ? fast_exp2(m - m_new) : 1.f;
      m = m_new;
      // Rescale this half's columns of O if the reference maximum moved.  O
      // is stable: S(j) was committed after P.V(j-1), and its arrival is what
      // this tile started on.
      if (j > 0 && __any_sync(0xffffffffu, bump)) {
#pragma unroll 1
        for (int c = 0; c < D / 2; c += 16) {        // this half's D/2 columns
          uint32_t o[16];
          const uint32_t oc = tOx + half * (D / 2) + c;
          tmem_load16(oc, o);
          uint32_t o8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) o8[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_store8(oc, o8);
#pragma unroll
          for (int i = 0; i < 8; ++i) o8[i] = __float_as_uint(__uint_as_float(o[8 + i]) * alpha);
          tmem_store8(oc + 8, o8);
        }
      }
      // pass 2: weights 2^(s*scale*log2e - m) -> tensor memory as fp16, and
      // the partial row sum.  32 scores at a time are read, and their 32
      // weights stored as 16 packed columns at the front of this half's
      // columns (keys 32c .. 32c+31 at columns 16c .. 16c+15): a store only
      // overwrites scores already read.  Pairs of keys use packed two-lane
      // fp32 instructions; one wait for all the stores.
      float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        tmem_load32(sj + c * 32, v);
        uint32_t hp[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int k = c * 32 + 2 * i;
          float x0, x1;
          ffma2(x0, x1, __uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]), sl2, sl2,
                -m_new, -m_new);
          float p0 = fast_exp2(x0);
          float p1 = fast_exp2(x1);
          if (diag) {
            p0 = kh0 + k <= pos ? p0 : 0.f;
            p1 = kh0 + k + 1 <= pos ? p1 : 0.f;
          }
          hp[i] = round_f16(p0, p1, &sum[(i & 1) * 2], &sum[(i & 1) * 2 + 1]);
        }
        tmem_store16_async(sj + c * 16, hp);
      }
      tmem_store_wait();
      l = l * alpha + ((sum[0] + sum[1]) + (sum[2] + sum[3]));
      tc_fence_before();
      mbar_arrive(&p_full[x]);
    }
    if (ok) ok = __all_sync(0xffffffffu, pf_wait(&o_done[x], (n_tiles - 1) & 1, abort, p.wait_ns));
    if (ok) {
      // the row sum: this half's plus the other half's (one more pair phase)
      *slot(2, half) = l;
      mbar_arrive(pr_bar);
      ok = __all_sync(0xffffffffu, pf_wait(pr_bar, n_tiles & 1, abort, p.wait_ns));
    }
    // Epilogue: out = O / l.  A tile whose rows all belong to the chunk goes
    // through shared memory -- this tile's now idle ring (K for tile A, V for
    // tile B: every MMA that read it has completed once o_done arrived) -- in
    // the 128-byte-swizzled layout of the output tensor map, then out as TMA
    // stores of 32-column boxes, so each row is written with whole lines
    // instead of a 512-byte stride between lanes.  The last tile of a chunk,
    // which may end inside it, is stored row by row.
    const bool full_tile = tokx + p.tq <= C;
    uint8_t *ostage = x == 0 ? sK : sV;
    constexpr int OBOX = kPfRows * 128;           // one 32-column box of 128 rows
    float fin = 0.f;                              // sum of this thread's outputs
    if (ok) {
      tc_fence_after();
      l += *reinterpret_cast<volatile float *>(slot(2, 1 - half));
      const float inv = 1.f / l;
      float *dst = p.out + ((size_t)(q0 + tokx + t) * p.num_q_heads + kh * G + g) * D +
                   half * (D / 2);
#pragma unroll 1
      for (int c4 = 0; c4 < D / 32; ++c4) {
        uint32_t o[16];
        tmem_load16(tOx + half * (D / 2) + c4 * 16, o);
        const int col0 = half * (D / 2) + c4 * 16;     // first of these 16 columns
        uint8_t *box = ostage + (col0 >> 5) * OBOX + r * 128;
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const float4 val =
              make_float4(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv,
                          __uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
          if (row_ok) fin += (val.x + val.y) + (val.z + val.w);
          if (full_tile) {
            const int chunk = ((col0 & 31) + i) >> 2;   // 16-byte chunk within the box row
            *reinterpret_cast<float4 *>(box + ((chunk ^ (r & 7)) << 4)) = val;
          } else if (row_ok) {
            *reinterpret_cast<float4 *>(dst + c4 * 16 + i) = val;
          }
        }
      }
    }
    // A bf16 V value beyond fp16's range became infinite in the P.V (and a
    // non-finite q or K gives non-finite scores): the row's outputs are then
    // not finite, and so is their sum (the outputs of finite inputs are
    // bounded by max |v|, far from overflowing it).
    if (std::is_same<T, __nv_bfloat16>::value && !(fabsf(fin) <= 3.0e38f))
      flag_error(PA_DEVERR_RANGE);
    if (full_tile) {
      // every thread of the tile reaches this barrier, whether or not it
      // aborted: the branch above holds no early exit
      fence_proxy_async_smem();
      named_barrier_sync(1 + x, 256);
      if (warp == 2 + 8 * x && lane == 0 && !*abort) {
#pragma unroll 1
        for (int b = 0; b < D / 32; ++b)
          tma_store_3d(&omap, ostage + b * OBOX, b * 32, kh * G, q0 + tokx);
        bulk_commit_group();
        bulk_wait_group_read0();     // the ring is free once the stores read it
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kPfTmemCols);
  }
}

}  // namespace pa
