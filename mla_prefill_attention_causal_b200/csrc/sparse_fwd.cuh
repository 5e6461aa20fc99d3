// Absorbed top-k sparse MLA prefill forward for sm_100a.
//
// For token t and head h: O[t,h,:] = sum_r softmax_r(scale * q[t,h,:] .
// kv[idx[t,r], :]) * kv[idx[t,r], 0:512] over the valid slots r of the
// token's index list (the "SparseFlashMla" README, Description -- Formula,
// with K~ = V~ the selected rows; Parameters: -1 marks an invalid slot;
// Constraints: one index list per token shared by all heads), over the BF16
// latent cache of the Mojo "mla_prefill_branch_sparse_fp8" absorbed branch
// (576 = 512 latent + 64 rope dims; V is the first 512).
//
// All heads of a token share the selected rows, so the heads are the MMA's
// M dimension (128 rows; fewer heads are padded).  With 128 heads the
// output alone (128 x 512 fp32) would fill the whole TMEM, so each token is
// handled by two CTAs, CTA `half` producing value dims [256 half, +256);
// both compute the scores.  Per CTA (416 threads):
//   warps 0-3   softmax + epilogue (thread = head row = TMEM lane); they also
//               write Q dims [0, 256) into TMEM, the A operand of those MMAs
//   warps 4-11  loaders: the chunk's key rows (64 keys x 576 dims, 72 KB) are
//               copied with 16-byte cp.async, eight threads per row, into one
//               of two chunk slots laid out as the MMAs' 128-byte-swizzled
//               K-major tiles; padded slots are zero-filled without a read.
//               (Random 1152-byte rows stream several times faster this way
//               than through tile::gather4, whose issue rate caps one SM's
//               gather bandwidth well below what the tensor cores consume.)
//   warp  12    MMA issuer; also the TMA of Q dims [256, 576) into shared
//               memory
// TMEM (512 columns): S buffers [0,64) and [64,128) (P overwrites their
// first 32 columns), Q dims 0-255 as bf16 pairs [128,256), O [256,512).
// MMAs are issued as their inputs arrive; S of the next chunk runs while
// the current chunk's softmax does.  Chunks after the token's last valid
// slot are not processed.
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace mla {
namespace sparse {

constexpr int kM = 128;                          // heads per MMA (rows)
constexpr int kDl = 576;                         // 512 latent + 64 rope
constexpr int kDv = 512;
constexpr int kDvHalf = 256;                     // value dims per CTA
constexpr int kChunk = 64;                       // keys per chunk (MMA N of S)
constexpr int kUnits = kDl / 64;                 // 9 units of 64 dims per chunk
constexpr int kUnitBytes = kChunk * 128;         // 64 keys x 64 bf16 = 8 KB
constexpr int kSlotBytes = kUnits * kUnitBytes;  // 72 KB
constexpr int kSlots = 2;
constexpr int kQtDims = 256;                     // Q dims in TMEM
constexpr int kQsChunks = (kDl - kQtDims) / 64;  // 5 chunks of 128 rows x 64 dims
constexpr int kQChunkBytes = kM * 128;           // 16 KB
constexpr int kQsBytes = kQsChunks * kQChunkBytes;
constexpr int kLoadWarps = 8;
constexpr int kLoaders = 32 * kLoadWarps;
constexpr int kMmaWarp = 4 + kLoadWarps;
constexpr int kThreads = 32 * (kMmaWarp + 1);
constexpr int kTmemCols = 512;
constexpr int kColQ = 128;
constexpr int kColO = 256;

struct alignas(8) Bars {
  uint64_t q_full;          // TMA bytes of Q's shared-memory part
  uint64_t qt_ready;        // 4 softmax warps wrote Q's TMEM part
  uint64_t full[kSlots];    // every loader thread's copies of a chunk landed
  uint64_t empty[kSlots];   // the chunk's PV MMAs done
  uint64_t s_full[2];
  uint64_t p_full[2];       // 4 softmax warps
  uint64_t pv_done;         // one phase per PV(c)
  uint64_t o_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int last_valid;           // position of the token's last valid slot (-1: none)
};

constexpr int kSmemBytes = 1024 + kQsBytes + kSlots * kSlotBytes + static_cast<int>(sizeof(Bars));
static_assert(kSmemBytes <= 227 * 1024, "dynamic shared memory above the per-CTA limit");

struct Params {
  const __nv_bfloat16* q;  // [T, H, 576]
  const __nv_bfloat16* kv; // [N, 576]
  const int* indices;      // [T, topk]
  __nv_bfloat16* out;      // [T, H, 512]
  float* lse;              // [H, T] or null
  int num_tokens;
  int num_heads;
  int num_rows;
  int topk;
  float scale_log2;
  int wide_out;            // out is 32-byte aligned: every row half starts on a 32-byte boundary
  uint64_t timeout_ns;
};

constexpr uint32_t kIdescS = idesc_bf16_f32(128, kChunk, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kDvHalf, true);

__global__ void __launch_bounds__(kThreads, 1)
    sparse_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t = static_cast<int>(blockIdx.x >> 1);
  const int half = static_cast<int>(blockIdx.x & 1);

  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sQ = smem_u32(base);
  const uint32_t sRing = sQ + kQsBytes;
  Bars* bars = reinterpret_cast<Bars*>(base + kQsBytes + kSlots * kSlotBytes);
  volatile int* abort_flag = &bars->abort;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    mbar_init(smem_u32(&bars->qt_ready), 4);
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(smem_u32(&bars->full[i]), kLoaders);
      mbar_init(smem_u32(&bars->empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->s_full[i]), 1);
      mbar_init(smem_u32(&bars->p_full[i]), 4);
    }
    mbar_init(smem_u32(&bars->pv_done), 1);
    mbar_init(smem_u32(&bars->o_full), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort = 0;
    bars->last_valid = -1;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint64_t tlim = p.timeout_ns;
  auto warp_wait = [&](uint32_t bar, uint32_t parity, unsigned err) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, err, tlim));
  };

  // Prologue.  Q dims 256-575 go to shared memory by TMA and the softmax
  // warps write Q dims 0-255 into TMEM; meanwhile the other warps find the
  // last valid slot of the token's index list.  Chunks after it hold only
  // padding and are not processed (left-aligned lists with -1 fill, the
  // common layout, then skip all their padding; padding elsewhere is masked).
  if (warp == kMmaWarp && lane == 0) {
    prefetch_tensormap(&tm_q);
    mbar_arrive_expect_tx(smem_u32(&bars->q_full), kQsBytes);
    for (int c = 0; c < kQsChunks; ++c)
      tma_load_2d_hint(sQ + c * kQChunkBytes, &tm_q, kQtDims + 64 * c, t * p.num_heads,
                       smem_u32(&bars->q_full), l2_policy_evict_first());
  }
  if (warp < 4) {
    // Q dims 0-255 of this head as bf16 pairs in TMEM columns [kColQ, +128)
    const int h = threadIdx.x;
    const bool row_ok = h < p.num_heads;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint4* qrow = reinterpret_cast<const uint4*>(
        p.q + (static_cast<size_t>(t) * p.num_heads + (row_ok ? h : 0)) * kDl);
#pragma unroll
    for (int c = 0; c < kQtDims / 32; ++c) {  // 32 dims = 16 columns per store
      uint32_t v[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 w = row_ok ? __ldg(qrow + 4 * c + i) : make_uint4(0u, 0u, 0u, 0u);
        v[4 * i] = w.x;
        v[4 * i + 1] = w.y;
        v[4 * i + 2] = w.z;
        v[4 * i + 3] = w.w;
      }
      tmem_st_x16(tmem + lane_off + kColQ + 16 * c, v);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars->qt_ready));
  } else {
    // Each warp walks its positions from the end of the list backwards and
    // stops at its first valid slot (the largest of its positions), so an
    // unpadded list costs one load per thread.
    const int* idx_row = p.indices + static_cast<size_t>(t) * p.topk;
    constexpr int kScanThreads = kThreads - 128;
    const int r = static_cast<int>(threadIdx.x) - 128;
    int last = -1;
    for (int base = p.topk - kScanThreads; base > -kScanThreads; base -= kScanThreads) {
      const int i = base + r;
      int hit = -1;
      if (i >= 0) {
        const int v = __ldg(idx_row + i);
        if (v >= 0 && v < p.num_rows) hit = i;
      }
      hit = __reduce_max_sync(0xffffffffu, hit);
      if (hit >= 0) {
        last = hit;
        break;
      }
    }
    if (lane == 0 && last >= 0) atomicMax(&bars->last_valid, last);
  }
  __syncthreads();
  const int nchunks = (bars->last_valid + kChunk) / kChunk;  // chunks up to the last valid slot

  if (warp >= 4 && warp < kMmaWarp) {
    // ------------------------------------------------------------ loaders
    // Thread i copies 16-byte column j = i % 8 of every 64-dim unit of keys
    // i / 8 and i / 8 + 32; in the 128-byte swizzle that column of key k
    // sits at 16-byte position j ^ (k % 8) of the key's 128-byte row.
    const int li = threadIdx.x - 128;
    const int j = li & 7;
    const int k0 = li >> 3;  // 0..31
    const int* idx_row = p.indices + static_cast<size_t>(t) * p.topk;
    auto fetch = [&](int c, int r) -> int {
      const int key = c * kChunk + k0 + 32 * r;
      return key < p.topk ? __ldg(idx_row + key) : -1;
    };
    int vn0 = fetch(0, 0), vn1 = fetch(0, 1);
    for (int c = 0; c < nchunks; ++c) {
      const int slot = c % kSlots;
      const int v0 = vn0, v1 = vn1;
      if (c + 1 < nchunks) {  // next chunk's indices load while this one waits
        vn0 = fetch(c + 1, 0);
        vn1 = fetch(c + 1, 1);
      }
      if (!warp_wait(smem_u32(&bars->empty[slot]),
                     (static_cast<uint32_t>(c / kSlots) & 1u) ^ 1u, MLA_DEVSTAT_WAIT_TIMEOUT_LOAD))
        break;
      const uint32_t sbase = sRing + slot * kSlotBytes;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int v = r == 0 ? v0 : v1;
        const int k = k0 + 32 * r;
        const bool valid = v >= 0 && v < p.num_rows;
        const __nv_bfloat16* src = p.kv + static_cast<size_t>(valid ? v : 0) * kDl + 8 * j;
        const uint32_t dst = sbase + k * 128 + ((j ^ (k & 7)) << 4);
        const uint32_t nbytes = valid ? 16u : 0u;
#pragma unroll
        for (int u = 0; u < kUnits; ++u) cp_async_16(dst + u * kUnitBytes, src + 64 * u, nbytes);
      }
      cp_async_arrive_noinc(smem_u32(&bars->full[slot]));
    }
    cp_async_wait_all();  // never leave with copies into shared memory in flight
  } else if (warp == kMmaWarp) {
    // -------------------------------------------------------- MMA issuer
    bool ok = true;
    auto wait_bar = [&](uint32_t bar, uint32_t parity) -> bool {
      const bool r = warp_wait(bar, parity, MLA_DEVSTAT_WAIT_TIMEOUT_MMA);
      tc_fence_after();
      return r;
    };
    auto issue_s = [&](int c) {
      const int buf = c & 1;
      const uint32_t kv = sRing + (c % kSlots) * kSlotBytes;
      // dims 0-255: A = Q from TMEM
#pragma unroll 1
      for (int u = 0; u < kQtDims / 64; ++u) {
        mma_ts_x4_elect<2>(tmem + buf * kChunk, tmem + kColQ + u * 32,
                           sdesc_sw128(kv + u * kUnitBytes, 16, 1024), kIdescS, u > 0 ? 1u : 0u);
      }
      // dims 256-575: A = Q from shared memory
#pragma unroll 1
      for (int u = kQtDims / 64; u < kUnits; ++u) {
        mma_ss_x4_elect(tmem + buf * kChunk, sdesc_sw128(sQ + (u - kQtDims / 64) * kQChunkBytes, 16, 1024),
                        sdesc_sw128(kv + u * kUnitBytes, 16, 1024), kIdescS, 1u);
      }
      tc_commit_elect(smem_u32(&bars->s_full[buf]));
    };
    auto issue_pv = [&](int c) {
      const int buf = c & 1;
      // this CTA's value dims: units 4*half .. 4*half+3 (four 64-dim atoms, LBO 8 KB)
      const uint32_t vb = sRing + (c % kSlots) * kSlotBytes + 4 * half * kUnitBytes;
      // four MMAs of 16 keys (16 key rows of 128 bytes) each
      mma_ts_x4_elect<128>(tmem + kColO, tmem + buf * kChunk, sdesc_sw128(vb, kUnitBytes, 1024),
                           kIdescPV, c > 0 ? 1u : 0u);
      tc_commit_elect(smem_u32(&bars->pv_done));
      tc_commit_elect(smem_u32(&bars->empty[c % kSlots]));
    };
    ok = wait_bar(smem_u32(&bars->q_full), 0) && wait_bar(smem_u32(&bars->qt_ready), 0);
    // Issue S(c) and PV(c) in whichever order their inputs arrive: PV(c)
    // frees chunk c's slot for the next gather, so it must not queue behind
    // the wait for a later chunk's rows.  S(c) reuses the S/P buffer of
    // chunk c-2, so it follows PV(c-2) in issue order.
    auto ready = [&](uint32_t bar, uint32_t parity) -> bool {
      return __shfl_sync(0xffffffffu, lane == 0 ? mbar_test_wait(bar, parity) : 0u, 0) != 0u;
    };
    int s_next = 0, pv_next = 0;
    uint64_t t_last = globaltimer_ns();
    while (ok && pv_next < nchunks) {
      bool progressed = false;
      if (pv_next < s_next &&
          ready(smem_u32(&bars->p_full[pv_next & 1]), static_cast<uint32_t>(pv_next >> 1) & 1u)) {
        if (!(ok = wait_bar(smem_u32(&bars->p_full[pv_next & 1]),
                            static_cast<uint32_t>(pv_next >> 1) & 1u)))
          break;
        issue_pv(pv_next++);
        progressed = true;
      }
      if (s_next < nchunks && s_next <= pv_next + 1 &&
          ready(smem_u32(&bars->full[s_next % kSlots]),
                static_cast<uint32_t>(s_next / kSlots) & 1u)) {
        if (!(ok = wait_bar(smem_u32(&bars->full[s_next % kSlots]),
                            static_cast<uint32_t>(s_next / kSlots) & 1u)))
          break;
        fence_proxy_async_smem();  // the rows landed through the generic proxy
        issue_s(s_next++);
        progressed = true;
      }
      if (progressed) {
        t_last = globaltimer_ns();
      } else {
        if (*abort_flag) {
          ok = false;
        } else if (globaltimer_ns() - t_last > tlim) {
          if (lane == 0) {
            *abort_flag = 1;
            atomicOr(&g_mla_status, MLA_DEVSTAT_WAIT_TIMEOUT_MMA);
          }
          ok = false;
        }
        ok = __all_sync(0xffffffffu, ok);
        __nanosleep(8);
      }
    }
    tc_commit_elect(smem_u32(&bars->o_full));
    tc_commit_elect(smem_u32(&bars->drain));
    __syncwarp();
    volatile int no_abort = 0;
    mbar_wait(smem_u32(&bars->drain), 0, &no_abort, MLA_DEVSTAT_WAIT_TIMEOUT_MMA, tlim);
    // the Q copy has landed unless a wait gave up before it was seen
    mbar_wait(smem_u32(&bars->q_full), 0, &no_abort, MLA_DEVSTAT_WAIT_TIMEOUT_MMA, tlim);
  } else {
    // ---------------------------------------------- softmax + epilogue
    const int h = threadIdx.x;  // head row = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const bool row_ok = h < p.num_heads;
    const float sl2 = p.scale_log2;
    const uint64_t c2 = pack_f32x2(sl2, sl2);
    const Exp2PolyConsts pk2 = exp2_poly_consts();
    float m_run = -INFINITY;
    float l_run = 0.0f;
    bool ok = true;
    const int* idx_row = p.indices + static_cast<size_t>(t) * p.topk;
    for (int c = 0; c < nchunks; ++c) {
      const int buf = c & 1;
      const uint32_t tS = tmem + lane_off + buf * kChunk;
      // Which of the chunk's 64 slots hold a valid row: each warp reads the
      // index list itself (two entries per lane); the loads complete while
      // the warp waits for S.
      const int key_a = c * kChunk + lane, key_b = key_a + 32;
      const int ia = key_a < p.topk ? __ldg(idx_row + key_a) : -1;
      const int ib = key_b < p.topk ? __ldg(idx_row + key_b) : -1;
      if (!(ok = warp_wait(smem_u32(&bars->s_full[buf]), static_cast<uint32_t>(c >> 1) & 1u,
                           MLA_DEVSTAT_WAIT_TIMEOUT_SOFTMAX)))
        break;
      const uint64_t vmask =
          static_cast<uint64_t>(__ballot_sync(0xffffffffu, ia >= 0 && ia < p.num_rows)) |
          (static_cast<uint64_t>(__ballot_sync(0xffffffffu, ib >= 0 && ib < p.num_rows)) << 32);
      tc_fence_after();
      uint32_t sraw[64];
      tmem_ld_x32_wait(tS, *reinterpret_cast<uint32_t(*)[32]>(&sraw[0]));
      tmem_ld_x32_wait(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sraw[32]));
      float x[64];
#pragma unroll
      for (int j = 0; j < 64; ++j)
        x[j] = ((vmask >> j) & 1ull) ? __uint_as_float(sraw[j]) : -INFINITY;
      float m4[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
      for (int j = 4; j < 60; j += 8)
#pragma unroll
        for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], x[j + q], x[j + 4 + q]);
#pragma unroll
      for (int q = 0; q < 4; ++q) m4[q] = fmaxf(m4[q], x[60 + q]);
      const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      const float m_new = fmaxf(m_run, mx * sl2);
      // Lazy rescaling: keep the old maximum unless the new one exceeds it by 8.
      const bool need = m_new > m_run + 8.0f;
      float alpha = 1.0f;
      if (need) {
        alpha = ex2_approx(m_run - m_new);
        l_run *= alpha;
        m_run = m_new;
      }
      const float m_use = (m_run == -INFINITY) ? 0.0f : m_run;
      const uint64_t negm2 = pack_f32x2(-m_use, -m_use);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if ((j & 7) < 7)  // 14 of every 16 pairs on the MUFU unit, 2 on the FMA pipe
            pk[j] = softmax_pair_mufu(x[32 * cc + 2 * j], x[32 * cc + 2 * j + 1], c2, negm2,
                                      acc[j & 3]);
          else
            pk[j] = softmax_pair_poly(x[32 * cc + 2 * j], x[32 * cc + 2 * j + 1], c2, negm2, pk2,
                                      acc[j & 3]);
        }
        tmem_st_x16(tS + 16u * cc, pk);
      }
      l_run += (sum_f32x2(acc[0]) + sum_f32x2(acc[1])) + (sum_f32x2(acc[2]) + sum_f32x2(acc[3]));
      // O may only be rescaled once PV(c-1) has finished (PV(c) waits for p_full).
      if (c > 0) {
        if (!(ok = warp_wait(smem_u32(&bars->pv_done), static_cast<uint32_t>(c - 1) & 1u,
                             MLA_DEVSTAT_WAIT_TIMEOUT_SOFTMAX)))
          break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
          const uint32_t tO = tmem + lane_off + kColO;
#pragma unroll 1
          for (int q = 0; q < kDvHalf / 32; ++q) {
            uint32_t o[32];
            tmem_ld_x32_wait(tO + 32u * q, o);
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
            tmem_st_x32(tO + 32u * q, o);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[buf]));
    }

    // --------------------------------------------------------- epilogue
    if (ok && (ok = warp_wait(smem_u32(&bars->o_full), 0, MLA_DEVSTAT_WAIT_TIMEOUT_SOFTMAX))) {
      tc_fence_after();
      const bool seen = m_run != -INFINITY;  // some valid slot
      const float inv = seen ? 1.0f / l_run : 0.0f;
      __nv_bfloat16* orow = p.out + (static_cast<size_t>(t) * p.num_heads + h) * kDv + half * kDvHalf;
      const uint32_t tO = tmem + lane_off + kColO;
#pragma unroll 1
      for (int q = 0; q < kDvHalf / 32; ++q) {
        uint32_t o[32];
        tmem_ld_x32_wait(tO + 32u * q, o);
        if (row_ok) {
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)  // no valid slot: O = 0 (TMEM O may be unwritten)
            pk[j] = seen ? pack_bf16x2(__uint_as_float(o[2 * j]) * inv,
                                       __uint_as_float(o[2 * j + 1]) * inv)
                         : 0u;
          if (p.wide_out) {  // two 32-byte stores: whole L2 sectors
#pragma unroll
            for (int w = 0; w < 2; ++w)
              asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(
                               orow + 32 * q + 16 * w),
                           "r"(pk[8 * w]), "r"(pk[8 * w + 1]), "r"(pk[8 * w + 2]),
                           "r"(pk[8 * w + 3]), "r"(pk[8 * w + 4]), "r"(pk[8 * w + 5]),
                           "r"(pk[8 * w + 6]), "r"(pk[8 * w + 7])
                           : "memory");
          } else {
            uint4* orow4 = reinterpret_cast<uint4*>(orow + 32 * q);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              orow4[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
          }
        }
      }
      if (row_ok && half == 0 && p.lse != nullptr)
        p.lse[static_cast<size_t>(h) * p.num_tokens + t] =
            seen ? (m_run + lg2_approx(l_run)) * 0.69314718055994530942f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace sparse
}  // namespace mla
