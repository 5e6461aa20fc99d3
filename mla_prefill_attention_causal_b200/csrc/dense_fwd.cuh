// Dense varlen MLA prefill forward for sm_100a.
//
// Computes O = softmax(scale * Q K^T [+ bottom-right causal mask]) V and the
// natural-log LSE per (row, head), the formula of the "SparseFlashMla"
// README (Description -- Formula) applied to the packed varlen layout of the
// "Sgl project Sglang FA4 Interface" page (I/O Contract) with the MLA head
// dims of vLLM's flash_attn.py MLA prefill backend (qk 128 nope + 64 rope =
// 192, v 128, K/V expanded per head).
//
// One CTA owns one (sequence, 256-row query block, head) tile, split into
// two 128-row sub-tiles that share every K/V block:
//   warps 0-3  softmax for sub-tile 0 (thread = query row = TMEM lane)
//   warps 4-7  softmax for sub-tile 1
//   warp  8    TMA producer: Q once, then K/V chunks into an 8-slot ring
//   warp  9    MMA issuer (one thread): S = Q K^T and O += P V (tcgen05)
// Shared memory: Q 96 KB (2 sub-tiles x 3 chunks of 128 rows x 64 dims) and
// a ring of 8 chunks of 16 KB; every chunk is a 128-row x 128-byte tile with
// the 128-byte swizzle that both TMA and the MMA descriptors use.  A K block
// (128 keys x 192 dims) is 3 chunks, a V block (128 keys x 128 dims) 2.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512);
// P_i (bf16, 64 columns) overwrites the first half of S_i once S_i is read.
//
// MMA issue order per KV block n (so one sub-tile's softmax overlaps the
// other's MMAs): PV0(n), S0(n+1), PV1(n), S1(n+1).  Masking is applied only
// to blocks that are not fully visible (the diagonal and the ragged end).
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace mla {
namespace dense {

constexpr int kSubRows = 128;                        // MMA M (rows per sub-tile)
constexpr int kCtaRows = 256;                        // query rows per CTA
constexpr int kBlockKeys = 128;                      // keys per KV block
constexpr int kDqk = 192;
constexpr int kDv = 128;
constexpr int kChunkBytes = 128 * 128;               // 128 rows x 64 bf16
constexpr int kQkChunks = kDqk / 64;                 // 3
constexpr int kVChunks = kDv / 64;                   // 2
constexpr int kItemsPerBlock = kQkChunks + kVChunks; // 5 ring items per KV block
constexpr int kRing = 8;
constexpr int kQBytes = 2 * kQkChunks * kChunkBytes; // 96 KB
constexpr int kRingBytes = kRing * kChunkBytes;      // 128 KB
constexpr int kThreads = 320;
constexpr int kTmemCols = 512;

struct alignas(8) Bars {
  uint64_t q_full;
  uint64_t full[kRing];
  uint64_t empty[kRing];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

constexpr int kSmemBytes = 1024 + kQBytes + kRingBytes + static_cast<int>(sizeof(Bars));

struct Params {
  const int* cu_q;
  const int* cu_k;
  __nv_bfloat16* out;
  float* lse;
  int num_heads;
  int total_q;
  int causal;
  float scale_log2;     // softmax_scale * log2(e)
  uint64_t timeout_ns;  // limit for every barrier wait
};

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false);
constexpr uint32_t kIdescPV128 = idesc_bf16_f32(128, 128, true);
constexpr uint32_t kIdescPV64 = idesc_bf16_f32(128, 64, true);

// Number of keys (a prefix [0, n)) that any row of the sub-tile starting at
// row0 may see, and hence the KV blocks the sub-tile must visit.
__device__ __forceinline__ int sub_tile_keys(int row0, int Lq, int Lk, int causal) {
  if (row0 >= Lq) return 0;
  if (!causal) return Lk;
  const int last = min(row0 + kSubRows - 1, Lq - 1);
  return max(0, min(Lk, last + (Lk - Lq) + 1));
}

__device__ __forceinline__ void rescale_o_row(uint32_t tO, float alpha) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t o[32];
    tmem_ld_x32_wait(tO + 32u * c, o);
#pragma unroll
    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
    tmem_st_x32(tO + 32u * c, o);
  }
  tmem_wait_st();
}

__global__ void __launch_bounds__(kThreads, 1)
    dense_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.z;
  const int h = blockIdx.y;
  const int mb = gridDim.x - 1 - blockIdx.x;  // longest (causal) blocks first

  const int q_start = p.cu_q[b];
  const int Lq = p.cu_q[b + 1] - q_start;
  const int k_start = p.cu_k[b];
  const int Lk = p.cu_k[b + 1] - k_start;
  const int m0 = mb * kCtaRows;
  if (m0 >= Lq) return;  // uniform for the whole CTA
  const int off = Lk - Lq;
  const int nb0 = (sub_tile_keys(m0, Lq, Lk, p.causal) + kBlockKeys - 1) / kBlockKeys;
  const int nb1 = (sub_tile_keys(m0 + kSubRows, Lq, Lk, p.causal) + kBlockKeys - 1) / kBlockKeys;
  const int nblk = max(nb0, nb1);

  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sQ = smem_u32(base);
  const uint32_t sRing = sQ + kQBytes;
  Bars* bars = reinterpret_cast<Bars*>(base + kQBytes + kRingBytes);
  volatile int* abort_flag = &bars->abort;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(smem_u32(&bars->full[i]), 1);
      mbar_init(smem_u32(&bars->empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->s_full[i]), 1);
      mbar_init(smem_u32(&bars->p_full[i]), kSubRows);
      mbar_init(smem_u32(&bars->o_full[i]), 1);
    }
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint64_t tlim = p.timeout_ns;

  if (warp == 8) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0 && nblk > 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      const uint64_t pol_kv = l2_policy_evict_last();
      const uint64_t pol_q = l2_policy_evict_first();
      const uint32_t qbar = smem_u32(&bars->q_full);
      mbar_arrive_expect_tx(qbar, kQBytes);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int c = 0; c < kQkChunks; ++c)
          tma_load_2d_hint(sQ + (i * kQkChunks + c) * kChunkBytes, &tm_q, h * kDqk + 64 * c,
                           q_start + m0 + i * kSubRows, qbar, pol_q);
      int issued = 0;
      bool ok = true;
      for (int n = 0; n < nblk && ok; ++n) {
        for (int it = 0; it < kItemsPerBlock; ++it) {
          const int item = n * kItemsPerBlock + it;
          const int slot = item % kRing;
          const uint32_t round = static_cast<uint32_t>(item / kRing);
          if (!mbar_wait(smem_u32(&bars->empty[slot]), (round & 1u) ^ 1u, abort_flag,
                         MLA_DEVSTAT_WAIT_TIMEOUT_LOAD, tlim)) {
            ok = false;
            break;
          }
          const uint32_t fbar = smem_u32(&bars->full[slot]);
          mbar_arrive_expect_tx(fbar, kChunkBytes);
          if (it < kQkChunks)
            tma_load_2d_hint(sRing + slot * kChunkBytes, &tm_k, h * kDqk + 64 * it,
                             k_start + n * kBlockKeys, fbar, pol_kv);
          else
            tma_load_2d_hint(sRing + slot * kChunkBytes, &tm_v, h * kDv + 64 * (it - kQkChunks),
                             k_start + n * kBlockKeys, fbar, pol_kv);
          ++issued;
        }
      }
      if (!ok) {
        // Unwinding: let the copies already issued land before the CTA exits.
        volatile int no_abort = 0;
        mbar_wait(qbar, 0, &no_abort, 0, tlim);
        const int first = max(0, issued - kRing);
        for (int item = first; item < issued; ++item) {
          mbar_wait(smem_u32(&bars->full[item % kRing]),
                    static_cast<uint32_t>(item / kRing) & 1u, &no_abort, 0, tlim);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------- MMA issuer
    if (nblk > 0) {
      auto wait_item = [&](int item) -> bool {
        return __all_sync(0xffffffffu,
                          mbar_wait(smem_u32(&bars->full[item % kRing]),
                                    static_cast<uint32_t>(item / kRing) & 1u, abort_flag,
                                    MLA_DEVSTAT_WAIT_TIMEOUT_MMA, tlim));
      };
      auto release_item = [&](int item) {
        if (lane == 0) tc_commit(smem_u32(&bars->empty[item % kRing]));
      };
      auto issue_s = [&](int i, int n) {
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < kDqk / 16; ++kk) {
            const int c = kk >> 2;
            const uint32_t koff = (kk & 3) * 32;
            const uint64_t a = sdesc_sw128(sQ + (i * kQkChunks + c) * kChunkBytes + koff, 16, 1024);
            const int slot = (n * kItemsPerBlock + c) % kRing;
            const uint64_t bd = sdesc_sw128(sRing + slot * kChunkBytes + koff, 16, 1024);
            mma_ss(tmem + i * 128, a, bd, kIdescQK, kk > 0 ? 1u : 0u);
          }
          tc_commit(smem_u32(&bars->s_full[i]));
        }
        __syncwarp();
      };
      auto issue_pv = [&](int i, int n) {
        if (lane == 0) {
          const int slot0 = (n * kItemsPerBlock + kQkChunks) % kRing;
          const int slot1 = (n * kItemsPerBlock + kQkChunks + 1) % kRing;
          const uint32_t tO = tmem + 256 + i * 128;
#pragma unroll
          for (int kk = 0; kk < kBlockKeys / 16; ++kk) {
            const uint32_t a_t = tmem + i * 128 + kk * 8;  // 16 bf16 of P = 8 columns
            const uint32_t acc = (n > 0 || kk > 0) ? 1u : 0u;
            const uint32_t koff = kk * 16 * 128;           // 16 key rows of 128 bytes
            if (slot1 == slot0 + 1) {
              const uint64_t bd = sdesc_sw128(sRing + slot0 * kChunkBytes + koff, kChunkBytes, 1024);
              mma_ts(tO, a_t, bd, kIdescPV128, acc);
            } else {
              const uint64_t b0 = sdesc_sw128(sRing + slot0 * kChunkBytes + koff, kChunkBytes, 1024);
              const uint64_t b1 = sdesc_sw128(sRing + slot1 * kChunkBytes + koff, kChunkBytes, 1024);
              mma_ts(tO, a_t, b0, kIdescPV64, acc);
              mma_ts(tO + 64, a_t, b1, kIdescPV64, acc);
            }
          }
        }
        __syncwarp();
      };
      auto wait_p = [&](int i, int n) -> bool {
        const bool ok = __all_sync(0xffffffffu,
                                   mbar_wait(smem_u32(&bars->p_full[i]), static_cast<uint32_t>(n) & 1u,
                                             abort_flag, MLA_DEVSTAT_WAIT_TIMEOUT_MMA, tlim));
        tc_fence_after();
        return ok;
      };

      bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->q_full), 0, abort_flag,
                                                  MLA_DEVSTAT_WAIT_TIMEOUT_MMA, tlim));
      for (int c = 0; c < kQkChunks && ok; ++c) ok = wait_item(c);
      if (ok) {
        tc_fence_after();
        if (nb0 > 0) issue_s(0, 0);
        if (nb1 > 0) issue_s(1, 0);
        for (int c = 0; c < kQkChunks; ++c) release_item(c);
      }
      for (int n = 0; n < nblk && ok; ++n) {
        const int vbase = n * kItemsPerBlock + kQkChunks;
        ok = wait_item(vbase) && wait_item(vbase + 1);
        if (!ok) break;
        tc_fence_after();
        if (n < nb0) {
          if (!(ok = wait_p(0, n))) break;
          issue_pv(0, n);
          if (n == nb0 - 1 && lane == 0) tc_commit(smem_u32(&bars->o_full[0]));
        }
        const bool more = n + 1 < nblk;
        if (more) {
          const int kbase = (n + 1) * kItemsPerBlock;
          ok = wait_item(kbase) && wait_item(kbase + 1) && wait_item(kbase + 2);
          if (!ok) break;
          tc_fence_after();
        }
        if (n + 1 < nb0) issue_s(0, n + 1);
        if (n < nb1) {
          if (!(ok = wait_p(1, n))) break;
          issue_pv(1, n);
          if (n == nb1 - 1 && lane == 0) tc_commit(smem_u32(&bars->o_full[1]));
        }
        if (more) {
          release_item(vbase);
          release_item(vbase + 1);
        }
        if (n + 1 < nb1) issue_s(1, n + 1);
        if (more) {
          const int kbase = (n + 1) * kItemsPerBlock;
          for (int c = 0; c < kQkChunks; ++c) release_item(kbase + c);
        }
      }
      // Wait until every MMA issued above has completed before the CTA ends.
      if (lane == 0) tc_commit(smem_u32(&bars->drain));
      __syncwarp();
      volatile int no_abort = 0;
      mbar_wait(smem_u32(&bars->drain), 0, &no_abort, MLA_DEVSTAT_WAIT_TIMEOUT_MMA, tlim);
    }
  } else {
    // ------------------------------------------------- softmax warpgroups
    const int sub = warp >> 2;
    const int wq = warp & 3;
    const int r = m0 + sub * kSubRows + wq * 32 + lane;  // row within the sequence
    const int row0 = m0 + sub * kSubRows;
    const int nb = sub == 0 ? nb0 : nb1;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + sub * 128;
    const uint32_t tO = tmem + lane_off + 256 + sub * 128;
    const int lim = p.causal ? min(Lk, r + off + 1) : Lk;  // keys [0, lim) visible
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;  // running max of scale*log2(e)*s (lazily updated)
    float l_run = 0.f;        // running sum of exp2(scaled s - m_run)
    bool ok = true;
    const uint32_t sbar = smem_u32(&bars->s_full[sub]);
    const uint32_t pbar = smem_u32(&bars->p_full[sub]);

    for (int n = 0; n < nb; ++n) {
      ok = __all_sync(0xffffffffu, mbar_wait(sbar, static_cast<uint32_t>(n) & 1u, abort_flag,
                                             MLA_DEVSTAT_WAIT_TIMEOUT_SOFTMAX, tlim));
      if (!ok) break;
      tc_fence_after();
      uint32_t sraw[128];
      tmem_ld_x128_wait(tS, sraw);
      float x[128];
#pragma unroll
      for (int j = 0; j < 128; ++j) x[j] = __uint_as_float(sraw[j]);
      const int kbase = n * kBlockKeys;
      const bool full_blk = (kbase + kBlockKeys <= Lk) &&
                            (!p.causal || kbase + kBlockKeys - 1 <= row0 + off);
      if (!full_blk) {
#pragma unroll
        for (int j = 0; j < 128; ++j)
          if (kbase + j >= lim) x[j] = -INFINITY;
      }
      float mx = x[0];
#pragma unroll
      for (int j = 1; j < 128; ++j) mx = fmaxf(mx, x[j]);
      const float m_new = fmaxf(m_run, mx * sl2);
      // Lazy rescaling: keep the old maximum unless the new one is larger by
      // more than 8 (a factor 256 in the exponentials, harmless in fp32/bf16).
      const bool need = m_new > m_run + 8.0f;
      float alpha = 1.0f;
      if (need) {
        alpha = ex2_approx(m_run - m_new);
        l_run *= alpha;
        m_run = m_new;
      }
      const float m_use = (m_run == -INFINITY) ? 0.0f : m_run;
      float sum = 0.0f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // 32 scores -> 16 packed bf16 pairs per store
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float p0 = ex2_approx(fmaf(x[32 * c + 2 * j], sl2, -m_use));
          const float p1 = ex2_approx(fmaf(x[32 * c + 2 * j + 1], sl2, -m_use));
          sum += p0 + p1;
          pk[j] = pack_bf16x2(p0, p1);
        }
        tmem_st_x16(tS + 16u * c, pk);
      }
      l_run += sum;
      // O(n-1) is complete (its MMAs precede S(n) in issue order) and PV(n)
      // waits for p_full, so O can be rescaled here, after the scores died.
      if (n > 0 && __any_sync(0xffffffffu, need)) rescale_o_row(tO, alpha);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(pbar);
    }

    // --------------------------------------------------------- epilogue
    const bool row_ok = r < Lq;
    const size_t row_index = static_cast<size_t>(q_start + r) * p.num_heads + h;
    uint4* orow = reinterpret_cast<uint4*>(p.out + row_index * kDv);
    float lse_val = -INFINITY;
    if (nb > 0 && ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->o_full[sub]), 0, abort_flag,
                                             MLA_DEVSTAT_WAIT_TIMEOUT_SOFTMAX, tlim));
    }
    if (nb > 0 && ok) {
      tc_fence_after();
      const float inv = l_run > 0.0f ? 1.0f / l_run : 0.0f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld_x32_wait(tO + 32u * c, o);
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          pk[j] = pack_bf16x2(__uint_as_float(o[2 * j]) * inv, __uint_as_float(o[2 * j + 1]) * inv);
        if (row_ok) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            orow[c * 4 + v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        }
      }
      if (l_run > 0.0f) lse_val = (m_run + lg2_approx(l_run)) * 0.69314718055994530942f;
    } else if (row_ok) {
#pragma unroll
      for (int v4 = 0; v4 < 16; ++v4) orow[v4] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (row_ok && p.lse != nullptr) p.lse[static_cast<size_t>(h) * p.total_q + q_start + r] = lse_val;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace dense
}  // namespace mla
