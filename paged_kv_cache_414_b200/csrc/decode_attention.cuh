// PagedAttention decode for sm_100a.
//
// What is computed ("Why OS Virtual Memory Paging Saved LLM Inference: The
// vLLM Breakthrough", section 2 "The PagedAttention Architecture"; "Can OS
// paging techniques reduce LLM serving memory waste?", second paragraph): for
// the newly generated token of every sequence, attention over the sequence's
// K/V, which lives in fixed-size blocks anywhere in a physical pool and is
// found through the sequence's block table, computed block by block.
//
// Work decomposition (a design for this GPU, not from the pages).  A "tile"
// is one (sequence s, kv head h, logical block j): B tokens of K and of V,
// B*D*2 bytes each.  Tiles are numbered in (s, h, j) order; the run of tiles
// of one (s, h) is a "segment".  The U tiles are cut into W equal contiguous
// ranges, one per warp of a grid that fills every SM, so every warp streams
// the same number of bytes whatever the length mix.  A warp keeps one online
// softmax state per segment; a segment that lies wholly inside one warp's
// range is written to `out` directly, a segment cut by range boundaries
// leaves one (max, sum, accumulator) partial per warp that touched it
// (split context), plus an 8-word descriptor of its range and first segment.
// A small merge kernel, launched as a programmatic dependent so its CTAs are
// resident and waiting when the streaming grid completes, combines the
// partials: one warp per (boundary between warp ranges, group of heads).
// The streaming kernel itself never waits on another warp, fences or takes
// an atomic.
//
// Data movement.  Each warp owns a ring of `nstage` shared-memory stages and
// issues its own copies: one 2-D TMA box per 64 head-dim columns of the K
// tile and of the V tile (128-byte swizzle, so the tensor-core fragment loads
// below are bank-conflict free), plus a 1-D bulk copy of the G query rows at
// the start of each segment.  Completion is counted in bytes on one mbarrier
// per stage; every wait is bounded in time.  Block ids are prefetched for up
// to 32 tiles ahead, one per lane.
//
// Arithmetic.  G = 1 (no grouped heads): fp32 FMA on CUDA cores, two lanes
// per token for q.K and one lane per 4 (or 2) head-dim columns for P.V.
// G >= 2: the G query heads of a group share every K/V tile, so q.K^T and
// P.V are small dense contractions: warp-level tensor-core MMA (m16n8k16,
// fp32 accumulate) with tokens as the M dimension of S^T = K Q^T and head-dim
// as the M dimension of O^T = V^T P^T; P is re-laid from accumulator to
// operand layout with movmatrix and fed as a hi + lo pair of 16-bit values so
// the product keeps ~fp32 accuracy.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include <type_traits>

#include "pa_device.cuh"

namespace pa {

constexpr uint64_t kDrainLimitNs = 20000000ull;    // 20 ms to drain after a time-out
constexpr int kMetaWords = 8;                      // per-warp descriptor for the merge

// Tile flags.
enum : int {
  TF_FIRST = 1,   // first tile of a segment in this warp's range
  TF_LAST = 2,    // last tile of a segment in this warp's range
  TF_J0 = 4,      // logical block 0 of the segment
  TF_JEND = 8,    // last logical block of the segment
  TF_SKIP = 16,   // block id out of range: no data, contributes nothing
  TF_NEWTOK = 32, // holds the sequence's newest token, which this call also writes
};

struct TileInfo {
  int s, h, j, valid, flags, nb, blk, pad;
  long long u;   // global tile index
};

struct DecodeParams {
  float *out;
  const uint8_t *q;
  // Fused cache write (decode step): the newest token of every sequence comes
  // from k_new / v_new [S, Hkv, D] and is also stored into the pool.  Null
  // for attention alone.
  const uint8_t *k_new;
  const uint8_t *v_new;
  uint8_t *k_cache_w;
  uint8_t *v_cache_w;
  const int32_t *block_tables;
  const int32_t *context_lens;
  long long *meta;     // [w_total][kMetaWords]: each warp's range and first segment
  float *part_ml;      // [2 * w_total][G][2]   (max in log2 units, sum)
  float *part_o;       // [2 * w_total][G][D]
  float scale_log2;    // scale * log2(e)
  int num_seqs, num_q_heads, num_kv_heads, group, head_dim;
  int max_blocks, num_blocks;
  int nstage;
  int min_tiles;       // fewest tiles a warp is given
  uint64_t wait_ns;    // limit of a wait on a copy before giving up (2 s by default)
};

__device__ __forceinline__ int ceil_div_i(int a, int b) { return (a + b - 1) / b; }

// L2 policy for data written now and read back by the next kernel: its lines
// are the last to be evicted.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Store of one float with an L2 cache policy.
__device__ __forceinline__ void st_global_hint(float *dst, float v, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(dst), "f"(v), "l"(policy)
               : "memory");
}

// Number of blocks of sequence s, with the length clamped into the table.
template <int B>
__device__ __forceinline__ int seq_blocks(const DecodeParams &p, int s, bool report) {
  int L = __ldg(p.context_lens + s);
  const int cap = p.max_blocks * B;
  if (L < 0 || L > cap) {
    if (report) flag_error(PA_DEVERR_CONTEXT_LEN);
    L = L < 0 ? 0 : cap;
  }
  return ceil_div_i(L, B);
}

template <int B>
__device__ __forceinline__ int seq_len_clamped(const DecodeParams &p, int s) {
  int L = __ldg(p.context_lens + s);
  const int cap = p.max_blocks * B;
  return L < 0 ? 0 : (L > cap ? cap : L);
}

// Smem byte offset of (row r, 16-byte chunk c of head-dim box `box`) inside a
// K or V tile laid out as D/64 boxes of [B rows][128 bytes] with the 128-byte
// swizzle (chunk index XOR row % 8).
template <int B>
__device__ __forceinline__ uint32_t swz(int box, int r, int c) {
  return (uint32_t)(box * (B * 128) + r * 128 + ((c ^ (r & 7)) << 4));
}

// ============================================================================
// G >= 2: tensor-core path.  NT = number of 8-wide head tiles (G <= 8*NT).
// ============================================================================
template <typename T, int D, int B, int NT>
struct MmaPath {
  static constexpr int KT = D / 16;   // k-steps of q.K^T, m-tiles of P.V
  static constexpr int MT = B / 16;   // token tiles per block
  float o[KT][NT][4];
  float m[NT][2];
  float l[NT][2];
  uint32_t qf[KT][NT][2];

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int a = 0; a < KT; ++a)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int r = 0; r < 4; ++r) o[a][n][r] = 0.f;
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        m[n][c] = -INFINITY;
        l[n][c] = 0.f;
      }
  }

  // B-operand fragments of Q^T from the staged query rows [G][D].
  __device__ __forceinline__ void load_q(const uint8_t *qs, int G, int lane) {
    const int g = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int head = n * 8 + g;
#pragma unroll
      for (int kk = 0; kk < KT; ++kk) {
        if (head < G) {
          const uint8_t *row = qs + head * (D * 2) + (kk * 16 + tig * 2) * 2;
          qf[kk][n][0] = *reinterpret_cast<const uint32_t *>(row);
          qf[kk][n][1] = *reinterpret_cast<const uint32_t *>(row + 16);
        } else {
          qf[kk][n][0] = 0u;
          qf[kk][n][1] = 0u;
        }
      }
    }
  }

  __device__ __forceinline__ void tile(uint32_t kb, uint32_t vb, int valid, float scale_log2,
                                       int lane) {
    const int g = lane >> 2, tig = lane & 3;
    const int mi = lane >> 3, ri = lane & 7;
    float sc[MT][NT][4];
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int r = 0; r < 4; ++r) sc[t][n][r] = 0.f;

    // S^T[token][head] = sum_d K[token][d] Q[head][d]
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      const int row = t * 16 + (mi & 1) * 8 + ri;
#pragma unroll
      for (int kk = 0; kk < KT; ++kk) {
        const int dim = kk * 16 + (mi >> 1) * 8;
        uint32_t a[4];
        ldmatrix_x4(a, kb + swz<B>(dim >> 6, row, (dim & 63) >> 3));
#pragma unroll
        for (int n = 0; n < NT; ++n) Mma<T>::run(sc[t][n], a, qf[kk][n][0], qf[kk][n][1]);
      }
    }

    // scale, mask the tokens past the sequence end, running max per head
    float mx[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n) mx[n][0] = mx[n][1] = -INFINITY;
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int tok = t * 16 + g + ((r & 2) ? 8 : 0);
          const float v = tok < valid ? sc[t][n][r] * scale_log2 : -INFINITY;
          sc[t][n][r] = v;
          mx[n][r & 1] = fmaxf(mx[n][r & 1], v);
        }
    float alpha[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float v = mx[n][c];
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
        const float mnew = fmaxf(m[n][c], v);
        alpha[n][c] = exp2f(m[n][c] - mnew);
        m[n][c] = mnew;
      }
    float ls[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n) ls[n][0] = ls[n][1] = 0.f;
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float pv = exp2f(sc[t][n][r] - m[n][r & 1]);
          sc[t][n][r] = pv;
          ls[n][r & 1] += pv;
        }
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int c = 0; c < 2; ++c) l[n][c] = l[n][c] * alpha[n][c] + ls[n][c];
#pragma unroll
    for (int a = 0; a < KT; ++a)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int r = 0; r < 4; ++r) o[a][n][r] *= alpha[n][r & 1];

    // O^T[d][head] += sum_token V[token][d] P[head][token]
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const uint32_t h01 = Mma<T>::pack(sc[t][n][0], sc[t][n][1]);
        const uint32_t h23 = Mma<T>::pack(sc[t][n][2], sc[t][n][3]);
        const float2 f01 = Mma<T>::unpack(h01), f23 = Mma<T>::unpack(h23);
        const uint32_t l01 = Mma<T>::pack(sc[t][n][0] - f01.x, sc[t][n][1] - f01.y);
        const uint32_t l23 = Mma<T>::pack(sc[t][n][2] - f23.x, sc[t][n][3] - f23.y);
        bh[n][0] = movmatrix_trans(h01);
        bh[n][1] = movmatrix_trans(h23);
        bl[n][0] = movmatrix_trans(l01);
        bl[n][1] = movmatrix_trans(l23);
      }
      // tokens of this thread's V fragments: t0 (+1) in a0/a1, t0+8 (+1) in a2/a3
      const int t0 = t * 16 + tig * 2;
      const bool tail = (t * 16 + 16) > valid;
      uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
      if (tail) {
        mlo = (t0 < valid ? 0x0000ffffu : 0u) | (t0 + 1 < valid ? 0xffff0000u : 0u);
        mhi = (t0 + 8 < valid ? 0x0000ffffu : 0u) | (t0 + 9 < valid ? 0xffff0000u : 0u);
      }
      const int vrow = t * 16 + (mi >> 1) * 8 + ri;
#pragma unroll
      for (int a = 0; a < KT; ++a) {
        const int dim = a * 16 + (mi & 1) * 8;
        uint32_t f[4];
        ldmatrix_x4_trans(f, vb + swz<B>(dim >> 6, vrow, (dim & 63) >> 3));
        f[0] &= mlo;
        f[1] &= mlo;
        f[2] &= mhi;
        f[3] &= mhi;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          Mma<T>::run(o[a][n], f, bh[n][0], bh[n][1]);
          Mma<T>::run(o[a][n], f, bl[n][0], bl[n][1]);
        }
      }
    }
  }

  // Write the segment: normalised output, or a partial for the merge.
  __device__ __forceinline__ void finish(const DecodeParams &p, int s, int h, bool complete,
                                         int slot, int lane) {
    const int g = lane >> 2, tig = lane & 3;
    const int G = p.group;
    float lt[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float v = l[n][c];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        lt[n][c] = v;
      }
    if (complete) {
      float *dst = p.out + ((int64_t)s * p.num_q_heads + (int64_t)h * G) * D;
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int head = n * 8 + tig * 2 + c;
          if (head < G) {
            const float inv = lt[n][c] > 0.f ? 1.f / lt[n][c] : 0.f;
#pragma unroll
            for (int a = 0; a < KT; ++a) {
              dst[head * D + a * 16 + g] = o[a][n][c] * inv;
              dst[head * D + a * 16 + g + 8] = o[a][n][2 + c] * inv;
            }
          }
        }
    } else {
      float *po = p.part_o + (int64_t)slot * G * D;
      float *pm = p.part_ml + (int64_t)slot * G * 2;
      // kept in L2 for the merge kernel that reads it next
      const uint64_t pol = l2_policy_evict_last();
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int head = n * 8 + tig * 2 + c;
          if (head < G) {
#pragma unroll
            for (int a = 0; a < KT; ++a) {
              st_global_hint(po + head * D + a * 16 + g, o[a][n][c], pol);
              st_global_hint(po + head * D + a * 16 + g + 8, o[a][n][2 + c], pol);
            }
            if (g == 0) {
              st_global_hint(pm + head * 2 + 0, m[n][c], pol);
              st_global_hint(pm + head * 2 + 1, lt[n][c], pol);
            }
          }
        }
    }
  }
};

// ============================================================================
// G == 1: CUDA-core path.
// ============================================================================
template <typename T, int D, int B>
struct ScalarPath {
  static constexpr int CPH = D / 16;   // 16-byte chunks per half row
  static constexpr int DPL = D / 32;   // head-dim columns per lane in P.V
  float acc[DPL];
  float m, l;
  float qr[D / 2];

  // Chunk (box, index in box) that a lane of the given half reads at step i.
  // D = 128: each half is one box; the order is rotated by 4 for the second
  // half so the two halves of a token never hit the same banks.
  __device__ __forceinline__ static void chunk(int i, int half, int &box, int &c) {
    if constexpr (D == 128) {
      box = half;
      c = (i + 4 * half) & 7;
    } else {
      box = 0;
      c = half * 4 + i;
    }
  }

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int k = 0; k < DPL; ++k) acc[k] = 0.f;
    m = -INFINITY;
    l = 0.f;
  }

  __device__ __forceinline__ void load_q(const uint8_t *qs, int /*G*/, int lane) {
    const int half = lane & 1;
#pragma unroll
    for (int i = 0; i < CPH; ++i) {
      int box, c;
      chunk(i, half, box, c);
      const uint4 v = *reinterpret_cast<const uint4 *>(qs + (box * 64 + c * 8) * 2);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = Mma<T>::unpack(w[e]);
        qr[i * 8 + 2 * e] = f.x;
        qr[i * 8 + 2 * e + 1] = f.y;
      }
    }
  }

  __device__ __forceinline__ void tile(const uint8_t *ks, const uint8_t *vs, int valid,
                                       float scale_log2, int lane) {
    const int tk = lane >> 1, half = lane & 1;
    constexpr int RR = B / 16;
    float sr[RR];
#pragma unroll
    for (int rr = 0; rr < RR; ++rr) {
      const int tok = rr * 16 + tk;
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < CPH; ++i) {
        int box, c;
        chunk(i, half, box, c);
        const uint4 v = *reinterpret_cast<const uint4 *>(ks + swz<B>(box, tok, c));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = Mma<T>::unpack(w[e]);
          dot = fmaf(qr[i * 8 + 2 * e], f.x, dot);
          dot = fmaf(qr[i * 8 + 2 * e + 1], f.y, dot);
        }
      }
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      sr[rr] = tok < valid ? dot * scale_log2 : -INFINITY;
    }
    float mx = sr[0];
#pragma unroll
    for (int rr = 1; rr < RR; ++rr) mx = fmaxf(mx, sr[rr]);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    const float mnew = fmaxf(m, mx);
    const float alpha = exp2f(m - mnew);
    m = mnew;
    float ps = 0.f;
#pragma unroll
    for (int rr = 0; rr < RR; ++rr) {
      sr[rr] = exp2f(sr[rr] - mnew);
      ps += sr[rr];
    }
    l = l * alpha + (half == 0 ? ps : 0.f);
#pragma unroll
    for (int k = 0; k < DPL; ++k) acc[k] *= alpha;

#pragma unroll
    for (int rr = 0; rr < RR; ++rr) {
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const int tok = rr * 16 + t;
        const float pt = __shfl_sync(0xffffffffu, sr[rr], 2 * t);
        if (tok < valid) {   // warp-uniform: never touch V past the end
          if constexpr (D == 128) {
            const uint2 v = *reinterpret_cast<const uint2 *>(
                vs + swz<B>(lane >> 4, tok, (lane & 15) >> 1) + (lane & 1) * 8);
            const float2 a = Mma<T>::unpack(v.x), b = Mma<T>::unpack(v.y);
            acc[0] = fmaf(pt, a.x, acc[0]);
            acc[1] = fmaf(pt, a.y, acc[1]);
            acc[2] = fmaf(pt, b.x, acc[2]);
            acc[3] = fmaf(pt, b.y, acc[3]);
          } else {
            const uint32_t v = *reinterpret_cast<const uint32_t *>(
                vs + swz<B>(0, tok, lane >> 2) + (lane & 3) * 4);
            const float2 a = Mma<T>::unpack(v);
            acc[0] = fmaf(pt, a.x, acc[0]);
            acc[1] = fmaf(pt, a.y, acc[1]);
          }
        }
      }
    }
  }

  __device__ __forceinline__ void finish(const DecodeParams &p, int s, int h, bool complete,
                                         int slot, int lane) {
    float lt = l;
#pragma unroll
    for (int x = 1; x < 32; x <<= 1) lt += __shfl_xor_sync(0xffffffffu, lt, x);
    if (complete) {
      float *dst = p.out + ((int64_t)s * p.num_q_heads + h) * D + lane * DPL;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      if constexpr (DPL == 4) {
        *reinterpret_cast<float4 *>(dst) =
            make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
      } else {
        *reinterpret_cast<float2 *>(dst) = make_float2(acc[0] * inv, acc[1] * inv);
      }
    } else {
      // kept in L2 for the merge kernel that reads it next
      float *po = p.part_o + (int64_t)slot * D + lane * DPL;
      const uint64_t pol = l2_policy_evict_last();
#pragma unroll
      for (int k = 0; k < DPL; ++k) st_global_hint(po + k, acc[k], pol);
      if (lane == 0) {
        st_global_hint(p.part_ml + (int64_t)slot * 2 + 0, m, pol);
        st_global_hint(p.part_ml + (int64_t)slot * 2 + 1, lt, pol);
      }
    }
  }
};

// ============================================================================
// Split-context merge, done by the last warp to finish a split segment.
// ============================================================================

// First tile of warp c when U tiles are cut into wa equal ranges, and the
// warp whose range holds tile u.
__device__ __forceinline__ long long warp_start(long long c, long long U, long long wa) {
  return c * U / wa;
}
__device__ __forceinline__ long long warp_of(long long u, long long U, long long wa) {
  return ((u + 1) * wa - 1) / U;
}

// Partial slot of part c (a warp) of the split segment that starts at tile lo.
__device__ __forceinline__ long long part_slot(long long c, long long lo, long long U,
                                               long long wa) {
  return (lo <= warp_start(c, U, wa)) ? 2 * c : 2 * c + 1;
}

// ============================================================================
// Launch plan, computed by every CTA from the context lengths alone: the total
// number of tiles U = Hkv * sum_s ceil(L_s / B), the number of active warps
// (at most w_total, at least p.min_tiles tiles each), and for each of NQ query
// tiles query(k, U, w_active) (negative = none) the sequence holding it, the
// sequence's first tile and its (clamped) length.  With zero_rows set, the
// output rows of empty sequences are zeroed (each by one CTA) and bad lengths
// reported.  All threads of the CTA must call it; it ends with __syncthreads.
// ============================================================================
template <int B, int NW, typename Query>
__device__ void cta_plan(const DecodeParams &p, long long w_total, Query query, bool zero_rows,
                         long long *red, int *loc_s, long long *loc_base, int *loc_L,
                         long long &U, long long &w_active) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int S = p.num_seqs, Hkv = p.num_kv_heads;
  constexpr int NT_ = NW * 32;   // threads per CTA
  constexpr int KMAX = 8;   // sequences per thread on the one-pass path
  U = 0;
  w_active = 0;
  auto set_ranges = [&](long long tot) {
    U = tot * Hkv;
    w_active = 0;
    if (U > 0) {
      w_active = (U + p.min_tiles - 1) / p.min_tiles;
      if (w_active > w_total) w_active = w_total;
    }
  };
  auto warp_u0 = [&](int k) -> long long { return query(k, U, w_active); };
  const int D = p.head_dim;
  auto zero_row = [&](int s) {   // empty sequence: zero output rows
    if (!zero_rows) return;
    float4 *row = reinterpret_cast<float4 *>(p.out + (int64_t)s * p.num_q_heads * D);
    for (int k = 0; k < p.num_q_heads * D / 4; ++k) row[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  };
  const int cap = p.max_blocks * B;
  if (S <= NT_ * KMAX) {
    // one pass: thread t owns sequences [t*K, t*K + K)
    const int K = (S + NT_ - 1) / NT_;
    const int sbeg = threadIdx.x * K;
    int Lr[KMAX];
#pragma unroll
    for (int k = 0; k < KMAX; ++k)
      Lr[k] = (k < K && sbeg + k < S) ? __ldg(p.context_lens + sbeg + k) : 0;
    int mine = 0;
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      if (k < K && sbeg + k < S) {
        int L = Lr[k];
        if (L < 0 || L > cap) {
          if (zero_rows && blockIdx.x == 0) flag_error(PA_DEVERR_CONTEXT_LEN);
          L = L < 0 ? 0 : cap;
        }
        Lr[k] = L;
        mine += ceil_div_i(L, B);
        if (L == 0 && ((sbeg + k) % gridDim.x) == blockIdx.x) zero_row(sbeg + k);
      }
    }
    int incl = mine;
#pragma unroll
    for (int x = 1; x < 32; x <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, x);
      if (lane >= x) incl += v;
    }
    if (lane == 31) red[warp] = incl;
    __syncthreads();
    long long before_warp = 0, tot = 0;
#pragma unroll
    for (int k = 0; k < NW; ++k) {
      if (k < warp) before_warp += red[k];
      tot += red[k];
    }
    set_ranges(tot);
    long long cum = before_warp + incl - mine;   // blocks before sequence sbeg
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
      if (k < K && sbeg + k < S) {
        const int nb = ceil_div_i(Lr[k], B);
        if (nb > 0) {
          const long long lo = cum * Hkv, hi = (cum + nb) * Hkv;
          for (int kk = 0; kk < NW; ++kk) {
            const long long uk = warp_u0(kk);
            if (uk >= lo && uk < hi) {
              loc_s[kk] = sbeg + k;
              loc_base[kk] = lo;
              loc_L[kk] = Lr[k];
            }
          }
        }
        cum += nb;
      }
    }
  } else {
    // many sequences: a pass for the total, then a chunked scan
    long long mine = 0;
    for (int s = threadIdx.x; s < S; s += NT_) {
      const int nb = seq_blocks<B>(p, s, zero_rows && blockIdx.x == 0);
      mine += nb;
      if (nb == 0 && (s % gridDim.x) == blockIdx.x) zero_row(s);
    }
#pragma unroll
    for (int x = 16; x > 0; x >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, x);
    if (lane == 0) red[warp] = mine;
    __syncthreads();
    long long tot = 0;
#pragma unroll
    for (int k = 0; k < NW; ++k) tot += red[k];
    set_ranges(tot);
    long long cta_max_u0 = -1;
    for (int k = 0; k < NW; ++k) cta_max_u0 = max(cta_max_u0, warp_u0(k));
    if (cta_max_u0 >= 0) {
      long long run = 0;
      for (int c0 = 0; c0 < S; c0 += NT_) {
        const int s = c0 + threadIdx.x;
        const int L = s < S ? seq_len_clamped<B>(p, s) : 0;
        const int nb = ceil_div_i(L, B);
        int incl = nb;
#pragma unroll
        for (int x = 1; x < 32; x <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, x);
          if (lane >= x) incl += v;
        }
        __syncthreads();
        if (lane == 31) red[warp] = incl;
        __syncthreads();
        long long before_warp = 0, chunk_tot = 0;
#pragma unroll
        for (int k = 0; k < NW; ++k) {
          if (k < warp) before_warp += red[k];
          chunk_tot += red[k];
        }
        const long long before = run + before_warp + incl - nb;   // blocks before seq s
        if (nb > 0) {
          const long long lo = before * Hkv, hi = (before + nb) * Hkv;
          for (int kk = 0; kk < NW; ++kk) {
            const long long uk = warp_u0(kk);
            if (uk >= lo && uk < hi) {
              loc_s[kk] = s;
              loc_base[kk] = lo;
              loc_L[kk] = L;
            }
          }
        }
        run += chunk_tot;
        if (run * Hkv > cta_max_u0) break;
      }
    }
  }
  __syncthreads();
}

// ============================================================================
// The attention kernel.
// ============================================================================

// Lane-parallel description of up to 32 consecutive tiles of one sequence.
struct TileBatch {
  int s, L, nb;      // warp-uniform
  int n;             // number of tiles in the batch (0 = none)
  int my_h, my_j, my_id;   // this lane's tile
};

template <int B>
__device__ __forceinline__ void make_batch(const DecodeParams &p, TileBatch &tb, int s, int L,
                                           int nb, int h, int j, int64_t remaining, int lane) {
  tb.s = s;
  tb.L = L;
  tb.nb = nb;
  const int64_t left_in_seq = (int64_t)p.num_kv_heads * nb - ((int64_t)h * nb + j);
  int64_t n = left_in_seq < remaining ? left_in_seq : remaining;
  tb.n = n < 32 ? (int)n : 32;
  tb.my_h = 0;
  tb.my_j = 0;
  tb.my_id = -1;
  if (lane < tb.n) {
    const int pos = h * nb + j + lane;
    tb.my_h = pos / nb;
    tb.my_j = pos - tb.my_h * nb;
    tb.my_id = __ldg(p.block_tables + (int64_t)s * p.max_blocks + tb.my_j);
  }
}

template <typename T, int D, int B, int NT, int NW>
__global__ void __launch_bounds__(NW * 32, NT == 0 ? 3 : 2)
    paged_decode_kernel(const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap, const DecodeParams p) {
  constexpr int TILE = B * D * 2;
  constexpr int STAGE = 2 * TILE;
  const int G = p.group;
  const int qbytes = G * D * 2;
  const int qstride = qbytes + 4 * D;   // query rows, then the new K and V rows
  const int nstage = p.nstage;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.num_seqs, Hkv = p.num_kv_heads;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // per-warp regions
  uint8_t *stages = smem + (size_t)warp * nstage * STAGE;
  uint8_t *qslots = smem + (size_t)NW * nstage * STAGE + (size_t)warp * nstage * qstride;
  TileInfo *info = reinterpret_cast<TileInfo *>(smem + (size_t)NW * nstage * (STAGE + qstride)) +
                   warp * nstage;
  uint64_t *bars = reinterpret_cast<uint64_t *>(
                       smem + (size_t)NW * nstage * (STAGE + qstride + sizeof(TileInfo))) +
                   warp * nstage;

  __shared__ long long red[NW];
  __shared__ int loc_s[NW];
  __shared__ long long loc_base[NW];
  __shared__ int loc_L[NW];

  if (threadIdx.x == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  if (lane == 0)
    for (int k = 0; k < nstage; ++k) mbar_init(&bars[k], 1);
  // Launched as a programmatic dependent of the previous kernel on the
  // stream: everything above overlaps its tail; nothing below may run before
  // its writes (the step's new K/V, say) are visible.
  grid_dependency_wait();
  allow_dependent_launch();   // the split merge may be scheduled meanwhile

  // ---- plan: total tiles, this CTA's warp ranges ---------------------------
  const long long w_total = (long long)gridDim.x * NW;
  const long long w = (long long)blockIdx.x * NW + warp;
  long long U = 0, w_active = 0;
  cta_plan<B, NW>(
      p, w_total, [&](int k, long long U_, long long wa_) -> long long {
        const long long wk = (long long)blockIdx.x * NW + k;   // first tile of warp k
        return wk < wa_ ? (wk * U_) / wa_ : -1;
      },
      true, red, loc_s, loc_base, loc_L, U, w_active);
  __syncthreads();
  if (lane == 0) fence_barrier_init();
  __syncwarp();
  const bool active = w < w_active;
  const long long u0 = active ? (w * U) / w_active : 0;
  const long long u1 = active ? ((w + 1) * U) / w_active : 0;
  long long *meta = p.meta + w * kMetaWords;
  if (!active && lane < kMetaWords) meta[lane] = lane == 3 ? U : (lane == 4 ? w_active : 0);

  if (!active) return;

  // ---- this warp's first tile -----------------------------------------------
  const int s0 = loc_s[warp];
  const long long base0 = loc_base[warp];
  const int L0 = loc_L[warp];
  const int nb0 = ceil_div_i(L0, B);
  const long long r0 = u0 - base0;
  const int h0 = (int)(r0 / nb0);
  const int j0 = (int)(r0 - (long long)h0 * nb0);
  if (lane < kMetaWords) {   // descriptor: u0, first segment [lo, hi), U, active warps, s, h
    const long long seg_lo = base0 + (long long)h0 * nb0;
    long long v = 1;
    switch (lane) {
      case 0: v = u0; break;
      case 1: v = seg_lo; break;
      case 2: v = seg_lo + nb0; break;
      case 3: v = U; break;
      case 4: v = w_active; break;
      case 5: v = s0; break;
      case 6: v = h0; break;
      default: v = 1;
    }
    meta[lane] = v;
  }
  const long long ntiles = u1 - u0;

  // ---- issue cursor ---------------------------------------------------------
  TileBatch cur, nxt;
  long long issued = 0;          // tiles issued so far
  int cur_k = 0;                 // next tile of `cur` to issue
  make_batch<B>(p, cur, s0, L0, nb0, h0, j0, ntiles, lane);
  auto follow = [&](const TileBatch &b, long long remaining_after) {
    // the batch that comes after b in the walk
    TileBatch r;
    r.n = 0;
    r.s = b.s; r.L = b.L; r.nb = b.nb; r.my_h = 0; r.my_j = 0; r.my_id = -1;
    if (remaining_after <= 0) return r;
    const int last_h = __shfl_sync(0xffffffffu, b.my_h, b.n - 1);
    const int last_j = __shfl_sync(0xffffffffu, b.my_j, b.n - 1);
    int h = last_h, j = last_j + 1;
    int s = b.s, L = b.L, nb = b.nb;
    if (j == nb) { j = 0; ++h; }
    while (h >= Hkv || nb == 0) {   // next sequence with tiles
      ++s;
      if (s >= S) return r;
      L = seq_len_clamped<B>(p, s);
      nb = ceil_div_i(L, B);
      h = 0;
      j = 0;
    }
    make_batch<B>(p, r, s, L, nb, h, j, remaining_after, lane);
    return r;
  };
  nxt = follow(cur, ntiles - cur.n);

  const uint8_t *qbase = p.q;
  // K/V tiles are read once per call: evict them from L2 first, and the
  // partials this call writes for the split merge (evict-last) last.
  const uint64_t stream_policy = l2_policy_evict_first();
  auto issue = [&](int stage) {
    if (cur_k == cur.n) {
      cur = nxt;
      cur_k = 0;
      nxt = follow(cur, ntiles - issued - cur.n);
    }
    const int h = __shfl_sync(0xffffffffu, cur.my_h, cur_k);
    const int j = __shfl_sync(0xffffffffu, cur.my_j, cur_k);
    const int id = __shfl_sync(0xffffffffu, cur.my_id, cur_k);
    if (lane == 0) {
      int flags = 0;
      if (j == 0 || issued == 0) flags |= TF_FIRST;
      if (j == cur.nb - 1 || issued == ntiles - 1) flags |= TF_LAST;
      if (j == 0) flags |= TF_J0;
      if (j == cur.nb - 1) flags |= TF_JEND;
      const bool ok = id >= 0 && id < p.num_blocks;
      if (!ok) {
        flags |= TF_SKIP;
        flag_error(PA_DEVERR_BLOCK_ID);
      }
      if (ok && p.k_new != nullptr && j == cur.nb - 1) flags |= TF_NEWTOK;
      const int valid = min(B, cur.L - j * B);
      TileInfo ti;
      ti.s = cur.s; ti.h = h; ti.j = j; ti.valid = valid; ti.flags = flags;
      ti.nb = cur.nb;
      ti.blk = id;
      ti.pad = 0;
      ti.u = u0 + issued;
      info[stage] = ti;
      const uint32_t bytes = (ok ? STAGE : 0) + ((flags & TF_FIRST) ? qbytes : 0) +
                             ((flags & TF_NEWTOK) ? 4 * D : 0);
      uint64_t *bar = &bars[stage];
      if (bytes) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, bytes);
        if (ok) {
          const int row = (id * Hkv + h) * B;
          uint8_t *kd = stages + (size_t)stage * STAGE;
#pragma unroll
          for (int bx = 0; bx < D / 64; ++bx) {
            tma_load_2d_hint(kd + bx * (B * 128), &kmap, bx * 64, row, bar, stream_policy);
            tma_load_2d_hint(kd + TILE + bx * (B * 128), &vmap, bx * 64, row, bar, stream_policy);
          }
        }
        if (flags & TF_FIRST)
          bulk_load(qslots + (size_t)stage * qstride,
                    qbase + ((int64_t)cur.s * p.num_q_heads + (int64_t)h * G) * (D * 2), qbytes,
                    bar);
        if (flags & TF_NEWTOK) {
          const int64_t row = ((int64_t)cur.s * Hkv + h) * (D * 2);
          bulk_load(qslots + (size_t)stage * qstride + qbytes, p.k_new + row, D * 2, bar);
          bulk_load(qslots + (size_t)stage * qstride + qbytes + 2 * D, p.v_new + row, D * 2, bar);
        }
      } else {
        mbar_arrive(bar);
      }
    }
    ++cur_k;
    ++issued;
  };

  const int pre = ntiles < nstage ? (int)ntiles : nstage;
  for (int k = 0; k < pre; ++k) issue(k);

  // ---- consume --------------------------------------------------------------
  using Path = typename std::conditional<NT == 0, ScalarPath<T, D, B>, MmaPath<T, D, B, (NT > 0 ? NT : 1)>>::type;
  Path st;
  st.reset();
  bool seg_from0 = false;
  int seg_index = 0;
  for (long long i = 0; i < ntiles; ++i) {
    const int stage = (int)(i % nstage);
    const uint32_t parity = (uint32_t)((i / nstage) & 1);
    if (!mbar_wait_bounded(&bars[stage], parity, p.wait_ns)) {
      if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
      // drain the copies still in flight -- this tile's and those issued
      // after it -- so that none lands after the warp has left
      for (long long k = i; k < issued; ++k)
        mbar_wait_bounded(&bars[k % nstage], (uint32_t)((k / nstage) & 1), kDrainLimitNs);
      return;
    }
    const TileInfo ti = info[stage];
    if (ti.flags & TF_FIRST) {
      st.reset();
      st.load_q(qslots + (size_t)stage * qstride, G, lane);
      seg_from0 = (ti.flags & TF_J0) != 0;
    }
    if (ti.flags & TF_NEWTOK) {
      // the newest token: patch its K and V rows into the staged tile (the
      // pool still holds whatever was in that slot) and store them in the pool
      constexpr int CH = D / 8;   // 16-byte chunks per row
      const int r = ti.valid - 1;
      if (lane < 2 * CH) {
        const int isv = lane / CH, c = lane % CH;
        const uint4 v = *reinterpret_cast<const uint4 *>(qslots + (size_t)stage * qstride +
                                                         qbytes + isv * (2 * D) + c * 16);
        uint8_t *tile = stages + (size_t)stage * STAGE + isv * TILE;
        *reinterpret_cast<uint4 *>(tile + swz<B>(c >> 3, r, c & 7)) = v;
        uint8_t *pool = isv ? p.v_cache_w : p.k_cache_w;
        *reinterpret_cast<uint4 *>(pool + (((int64_t)ti.blk * Hkv + ti.h) * B + r) * (D * 2) +
                                   c * 16) = v;
      }
      __syncwarp();
    }
    if (!(ti.flags & TF_SKIP)) {
      const uint8_t *ks = stages + (size_t)stage * STAGE;
      if constexpr (NT == 0) {
        st.tile(ks, ks + TILE, ti.valid, p.scale_log2, lane);
      } else {
        st.tile(smem_addr(ks), smem_addr(ks + TILE), ti.valid, p.scale_log2, lane);
      }
    }
    if (ti.flags & TF_LAST) {
      const bool complete = seg_from0 && (ti.flags & TF_JEND);
      st.finish(p, ti.s, ti.h, complete, (int)(2 * w + (seg_index == 0 ? 0 : 1)), lane);
      ++seg_index;
    }
    __syncwarp();
    if (i + nstage < ntiles) issue(stage);
  }
}

// ============================================================================
// Merge of split segments.  Warp t of the grid handles boundary b = t / hc + 1
// between warp ranges b-1 and b, and heads [c*GMW, (c+1)*GMW) of the group,
// c = t % hc: if b is the first boundary inside the segment it cuts, the warp
// merges those heads' partials (several warps share a segment with many
// heads, so long segments with many partials are merged in parallel).
// Launched as a programmatic dependent of the streaming kernel.
// ============================================================================
template <int D, int GMW>
__global__ void __launch_bounds__(128, 6)
    paged_decode_merge_kernel(const DecodeParams p, int w_total, int hc) {
  constexpr int VPL = D / 32;
  constexpr int UNR = 16 / GMW;   // partials per batch of loads
  using VecT = typename std::conditional<VPL == 4, float4, float2>::type;
  grid_dependency_wait();
  const int lane = threadIdx.x & 31;
  const long long t = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
  const long long b = t / hc + 1;
  const int c = (int)(t % hc);
  if (b >= w_total) return;
  const long long mv = lane < kMetaWords ? __ldcg(p.meta + b * kMetaWords + lane)
                                         : __ldcg(p.meta + (b - 1) * kMetaWords);
  const long long ub = __shfl_sync(0xffffffffu, mv, 0);
  const long long lo = __shfl_sync(0xffffffffu, mv, 1);
  const long long hi = __shfl_sync(0xffffffffu, mv, 2);
  const long long U = __shfl_sync(0xffffffffu, mv, 3);
  const long long wa = __shfl_sync(0xffffffffu, mv, 4);
  const int s = (int)__shfl_sync(0xffffffffu, mv, 5);
  const int h = (int)__shfl_sync(0xffffffffu, mv, 6);
  const long long active = __shfl_sync(0xffffffffu, mv, 7);
  const long long uprev = __shfl_sync(0xffffffffu, mv, 8);
  // merge only at the first boundary inside a cut segment
  if (!active || lo >= ub || lo < uprev) return;
  const int G = p.group;
  const int g0 = c * GMW;
  if (g0 >= G) return;

  const long long c_lo = warp_of(lo, U, wa), c_hi = warp_of(hi - 1, U, wa);
  const long long n = c_hi - c_lo + 1;
  float M[GMW], den[GMW], num[GMW][VPL];
#pragma unroll
  for (int g = 0; g < GMW; ++g) {
    M[g] = -INFINITY;
    den[g] = 0.f;
#pragma unroll
    for (int v = 0; v < VPL; ++v) num[g][v] = 0.f;
  }
  for (long long k0 = 0; k0 < n; k0 += 32) {
    const long long k = k0 + lane;
    const bool ok = k < n;
    const long long slot = ok ? part_slot(c_lo + k, lo, U, wa) : 0;
    const int cnt = (int)((n - k0) < 32 ? (n - k0) : 32);
    float wk[GMW];
#pragma unroll
    for (int g = 0; g < GMW; ++g) {
      const int head = g0 + g < G ? g0 + g : G - 1;
      const float mk = ok ? __ldcg(p.part_ml + (slot * G + head) * 2) : -INFINITY;
      const float lk = ok ? __ldcg(p.part_ml + (slot * G + head) * 2 + 1) : 0.f;
      float cm = mk;
#pragma unroll
      for (int x = 16; x > 0; x >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, x));
      const float Mn = fmaxf(M[g], cm);
      const float so = Mn == -INFINITY ? 0.f : exp2f(M[g] - Mn);
      wk[g] = (mk == -INFINITY) ? 0.f : exp2f(mk - Mn);
      float dl = wk[g] * lk;
#pragma unroll
      for (int x = 16; x > 0; x >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, x);
      den[g] = den[g] * so + dl;
#pragma unroll
      for (int v = 0; v < VPL; ++v) num[g][v] *= so;
      M[g] = Mn;
    }
    for (int j0 = 0; j0 < cnt; j0 += UNR) {
      VecT buf[UNR][GMW];
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int j = j0 + u < cnt ? j0 + u : cnt - 1;
        const long long sj = __shfl_sync(0xffffffffu, slot, j);
#pragma unroll
        for (int g = 0; g < GMW; ++g) {
          const int head = g0 + g < G ? g0 + g : G - 1;
          buf[u][g] = __ldcg(reinterpret_cast<const VecT *>(p.part_o + (sj * G + head) * D +
                                                            lane * VPL));
        }
      }
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int j = j0 + u;
#pragma unroll
        for (int g = 0; g < GMW; ++g) {
          float wj = __shfl_sync(0xffffffffu, wk[g], j < cnt ? j : 0);
          wj = j < cnt ? wj : 0.f;
          num[g][0] = fmaf(wj, buf[u][g].x, num[g][0]);
          num[g][1] = fmaf(wj, buf[u][g].y, num[g][1]);
          if constexpr (VPL == 4) {
            num[g][2] = fmaf(wj, reinterpret_cast<const float4 &>(buf[u][g]).z, num[g][2]);
            num[g][3] = fmaf(wj, reinterpret_cast<const float4 &>(buf[u][g]).w, num[g][3]);
          }
        }
      }
    }
  }
  float *dst = p.out + ((int64_t)s * p.num_q_heads + (int64_t)h * G) * D + lane * VPL;
#pragma unroll
  for (int g = 0; g < GMW; ++g) {
    const int head = g0 + g;
    if (head < G) {
      const float inv = den[g] > 0.f ? 1.f / den[g] : 0.f;
      if constexpr (VPL == 4) {
        *reinterpret_cast<float4 *>(dst + head * D) =
            make_float4(num[g][0] * inv, num[g][1] * inv, num[g][2] * inv, num[g][3] * inv);
      } else {
        *reinterpret_cast<float2 *>(dst + head * D) = make_float2(num[g][0] * inv, num[g][1] * inv);
      }
    }
  }
}

}  // namespace pa
