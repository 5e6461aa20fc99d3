// Dense varlen MLA prefill forward for sm_100a.
//
// Computes O = softmax(scale * Q K^T [+ bottom-right causal mask]) V and the
// natural-log LSE per (row, head), the formula of the "SparseFlashMla"
// README (Description -- Formula) applied to the packed varlen layout of the
// "Sgl project Sglang FA4 Interface" page (I/O Contract) with the MLA head
// dims of vLLM's flash_attn.py MLA prefill backend (qk 128 nope + 64 rope =
// 192, v 128, K/V expanded per head).
//
// The kernel runs on CTA pairs (clusters of 2 on one TPC) and issues M=256
// tcgen05 MMAs with cta_group::2: each CTA keeps its own 128 query rows of
// an MMA in shared memory and TMEM, while each K/V block is split between
// the two CTAs (CTA r holds keys [64r, 64r+64) of every K block and value
// dims [64r, 64r+64) of every V block).  Compared with one CTA per MMA this
// halves each SM's K/V traffic and the shared-memory operand bytes per MMA.
//
// Work unit ("tile"): (sequence, 512-row query block, head) = two M=256
// sub-tiles that share every K/V block.  The query blocks are aligned to the
// end of the sequence, so that a ragged first block holds the rows that see
// the fewest keys.  A planner kernel sorts the
// (sequence, query block) entries by their number of visible KV blocks,
// longest first, into the caller's workspace.  Tile t of the resulting list
// is taken head-major (all entries of head 0, then of head 1, ...), except
// for the last few heads -- enough for about three rounds of the clusters
// -- which are taken entry-major (the longest entry of each of those
// heads, then the next, ...): clusters running at the same time then share
// the K/V of few heads in L2, and the list ends with the shortest tiles of
// the call.  The persistent clusters take tiles
// dynamically: cluster c starts with tile c, and whenever its producer warp
// is ready for another tile it takes the next index from a counter in the
// workspace, so a cluster that finishes early takes more work (greedy list
// scheduling over a longest-first list).  The producer hands each tile's
// coordinates to the other roles of both CTAs through a small ring in
// shared memory.  Which cluster runs a tile does not change how the tile is
// computed, so the output stays bitwise deterministic.
//
// Roles inside each CTA (384 threads):
//   warps 0-3  softmax + epilogue, sub-tile 0 (thread = query row = TMEM lane)
//   warps 4-7  softmax + epilogue, sub-tile 1
//   warp  8    producer: TMA loads of this CTA's Q rows and K/V halves, whose
//              completion is counted on the leader CTA's barriers
//   warp  9    (leader CTA only) MMA issuer: S = Q K^T, O += P V
// Shared memory per CTA: Q 96 KB (2 sub-tiles x 3 chunks of 128 rows x 64
// dims), a K ring of 3 slots (this CTA's 64 keys x 192 dims = 3 units of
// 64 rows x 64 dims, 24 KB) and a V ring of 3 slots (128 keys x this CTA's
// 64 dims = 2 units, 16 KB), all with the 128-byte swizzle used by TMA and
// the MMA descriptors.  K(b) and V(b) land on one barrier (the MMA warp
// waits once per block); K(b) is freed after both S MMAs of block b, V(b)
// after both PV MMAs.  Q, K and V are read through 3-D (dim, head, row)
// tensor maps, so strided views need no copies.
// TMEM per CTA (512 columns): S0 [0,128) S1 [128,256) O0 [256,384) O1
// [384,512); P_i (bf16, 64 columns) overwrites the first half of S_i.
//
// MMA issue order per KV block n (so one sub-tile's softmax overlaps the
// other's MMAs): PV0(n), S0(n+1), PV1(n), S1(n+1), where block n+1 may be
// the first block of the next tile.  Masking is applied only to blocks that
// are not fully visible (the diagonal and the ragged end).
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace mla {
namespace dense {

constexpr int kCtaRows = 128;                        // rows of a sub-tile held by one CTA
constexpr int kSubRows = 256;                        // MMA M (rows per sub-tile, both CTAs)
constexpr int kTileRows = 512;                       // query rows per tile
constexpr int kBlockKeys = 128;                      // keys per KV block (MMA N of S)
constexpr int kHalfKeys = 64;                        // keys of a K block held by one CTA
constexpr int kDqk = 192;                            // qk width of the MLA dims 128 + 64
constexpr int kDv = 128;                             // value dims of one pass
constexpr int kHalfDv = 64;                          // value dims held by one CTA
constexpr int kQChunkBytes = 128 * 128;              // 128 rows x 64 bf16
constexpr int kUnitBytes = 64 * 128;                 // 64 rows x 64 bf16
constexpr int kVUnits = kBlockKeys / 64;             // V half: 128 keys x 64 dims
constexpr int kVSlotBytes = kVUnits * kUnitBytes;    // 16 KB: this CTA's half of a V block
constexpr int kThreads = 384;          // 3 warpgroups; warps 10-11 only hold registers
// Register split (setmaxnreg): launched at kLaunchRegs per thread, the two
// softmax warpgroups grow to kSoftmaxRegs and the producer/MMA warpgroup
// shrinks to kOtherRegs; 8*32*224 + 4*32*56 = 384*168, the launch's total.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 224;
constexpr int kOtherRegs = 56;
static_assert(8 * 32 * kSoftmaxRegs + 4 * 32 * kOtherRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kTmemCols = 512;
constexpr int kPlanThreads = 1024;
constexpr int kPlanBins = 4096;                      // work histogram bins (clamped)
constexpr int kTailRounds = 3;                       // rounds of clusters the entry-major tail spans
constexpr int kTileSlots = 4;                        // tiles in flight in the hand-off ring

// Workspace layout (caller-provided device memory, 16-byte aligned).
struct WsHeader {
  int num_entries;  // E: (sequence, 512-row block) entries
  int num_tiles;    // E * num_heads * nsplit
  int next_tile;    // tiles taken from the counter so far (reset by the planner)
  int pad;
};
constexpr size_t kWsHeaderBytes = 256;

// A tile: its sequence's queries, keys and (for a call with a context, see
// mla_prefill_fwd_context) context keys, the first query row, the head and,
// for a split-KV call, which of the splits of its KV blocks it covers
// (packed as hs = head | split << 16).  A tile always has query rows, so
// Lq == 0 marks "no tile" (the end of a cluster's list).
struct alignas(16) TileInfo {
  int q_start, Lq, k_start, Lk;
  int c_start, Lc, m0, hs;
  __host__ __device__ bool valid() const { return Lq > 0; }
  __host__ __device__ int head() const { return hs & 0xffff; }
  __host__ __device__ int split() const { return hs >> 16; }
};

template <int SLOTS>
struct alignas(16) Bars {
  TileInfo tiles[kTileSlots];     // both: tile hand-off ring (written by the leader's producer)
  static_assert(sizeof(TileInfo) == 32, "a ring slot is two 16-byte stores");
  uint64_t tile_full[kTileSlots];   // both: the slot holds the next tile
  uint64_t tile_empty[kTileSlots];  // leader: every reader of the slot is done with it
  uint64_t q_full[2];    // leader: both producers (and the Q bytes of both CTAs)
  uint64_t q_empty[2];   // both: last S MMA of the tile done
  uint64_t full_kv[SLOTS];   // leader: K- and V-half bytes of block b, both CTAs
  uint64_t empty_k[SLOTS];   // both: the S MMAs reading the K slot done
  uint64_t empty_v[SLOTS];   // both: the PV MMAs reading the V slot done
  uint64_t s_full[2];    // both
  uint64_t p_full[2];    // leader: 8 softmax warps (both CTAs)
  uint64_t o_full[2];    // both
  uint64_t o_empty[2];   // leader: 8 softmax warps (both CTAs)
  uint64_t drain;        // leader
  uint32_t tmem_base;
  int abort;
};

// Shared-memory plan for a qk width of DQK (128, 192 or 256) dims: Q of both
// sub-tiles (DQK/64 chunks of 128 rows x 64 dims each) and a ring of K/V
// block halves -- three slots, or two at DQK = 256, where Q alone takes
// 128 KB.  The value width of one pass is always 128 (kDv).
template <int DQK>
struct Geo {
  static_assert(DQK == 128 || DQK == 192 || DQK == 256, "qk width");
  static constexpr int kQkChunks = DQK / 64;
  static constexpr int kKUnits = kQkChunks;                   // K half: 64 keys x DQK dims
  static constexpr int kSlots = DQK == 256 ? 2 : 3;           // K and V blocks in flight
  static constexpr int kKSlotBytes = kKUnits * kUnitBytes;    // this CTA's half of a K block
  static constexpr int kQSubBytes = kQkChunks * kQChunkBytes;
  static constexpr int kQBytes = 2 * kQSubBytes;
  static constexpr int kRingBytes = kSlots * (kKSlotBytes + kVSlotBytes);
  static constexpr int kSmemBytes =
      1024 + kQBytes + kRingBytes + static_cast<int>(sizeof(Bars<kSlots>));
  static_assert(kSmemBytes <= 227 * 1024, "shared memory above the per-CTA limit");
};

struct Params {
  const int* cu_q;
  const int* cu_k;
  const int* cu_ctx;       // context keys per sequence ([batch + 1]), or null: no context
  void* out;               // bf16 [total_q, H, 128], or e4m3 when out_scale is set
  long long out_rs;        // row and head strides of out in elements (H * 128 and 128 for a
  long long out_hs;        // packed output; wider for one 128-dim pass of a wider value)
  float* lse;
  const float* sinks;      // one attention-sink logit per head, or null
  const float* out_scale;  // e4m3 output scale (device scalar), or null: bf16 output
  float* o_part;           // split-KV: fp32 [nsplit][total_q][H][128] partial outputs
  float* lse_part;         // split-KV: fp32 [nsplit][H][total_q] partial LSEs
  int wide_out;            // bit 0: every out row is 32-byte aligned; bit 1: every o_part row is
  int nsplit;              // KV splits per tile (1: none; the partials are unused)
  WsHeader* ws;
  const int2* entries;  // [E] {sequence, 512-row block index}, longest first
  int num_heads;
  int total_q;
  int causal;
  float scale_log2;     // softmax_scale * log2(e)
  uint64_t timeout_ns;  // limit for every barrier wait
};

constexpr uint32_t kIdescQK = idesc_bf16_f32(256, 128, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(256, 128, true);

// First row of a sequence's 512-row entry mb.  Entries are aligned to the
// end of the sequence (entry 0 holds its last 512 rows), so a ragged piece
// (Lq mod 512 rows) comes first, where rows see the fewest keys; its rows
// below 0 (and, in every entry, rows past Lq) are computed as masked filler
// and never stored.  With start-aligned entries the ragged piece would hold
// the last rows, whose sub-tile walks every KV block for a few rows.
__host__ __device__ __forceinline__ int entry_row0(int Lq, int mb) {
  return Lq - (mb + 1) * kTileRows;
}
// Number of keys (a prefix [0, n)) that any row of the 256-row sub-tile
// starting at row0 may see.
__host__ __device__ __forceinline__ int sub_tile_keys(int row0, int Lq, int Lk, int causal) {
  if (row0 >= Lq || row0 + kSubRows <= 0) return 0;
  if (!causal) return Lk;
  const int last = min(row0 + kSubRows - 1, Lq - 1);
  return max(0, min(Lk, last + (Lk - Lq) + 1));
}
__host__ __device__ __forceinline__ int blocks_for(int keys) {
  return (keys + kBlockKeys - 1) / kBlockKeys;
}
// KV blocks a 256-row sub-tile starting at row0 visits: every block of the
// sequence's context first (all context keys are visible), then the blocks
// of its own visible keys; none when it has no rows.
__host__ __device__ __forceinline__ int sub_tile_blocks(int row0, int Lq, int Lk, int Lc,
                                                        int causal) {
  if (row0 >= Lq || row0 + kSubRows <= 0) return 0;
  return blocks_for(Lc) + blocks_for(sub_tile_keys(row0, Lq, Lk, causal));
}
// Split-KV: a tile's block sequence (nmax = the longer sub-tile's blocks) is
// cut into nsplit ranges [s nmax / nsplit, (s+1) nmax / nsplit); split s of
// a sub-tile with n blocks visits blocks [lo, lo + count) of its own.
__host__ __device__ __forceinline__ int split_lo(int nmax, int s, int nsplit) {
  return static_cast<int>(static_cast<long long>(nmax) * s / nsplit);
}
__host__ __device__ __forceinline__ int split_count(int n, int nmax, int s, int nsplit) {
  const int lo = split_lo(nmax, s, nsplit), hi = split_lo(nmax, s + 1, nsplit);
  return max(0, min(hi, n) - lo);
}

// ------------------------------------------------------------------ planner
// One CTA: builds the (sequence, 512-row block) entry list sorted by the
// number of KV blocks its rows visit (descending).
__global__ void __launch_bounds__(kPlanThreads)
    dense_plan_kernel(const int* cu_q, const int* cu_k, const int* cu_ctx, int batch,
                      int causal, WsHeader* ws, int2* entries, int capacity, int num_heads,
                      int nsplit) {
  __shared__ int bins[kPlanBins];
  __shared__ int s_total;
  const int tid = threadIdx.x;
  for (int i = tid; i < kPlanBins; i += blockDim.x) bins[i] = 0;
  if (tid == 0) s_total = 0;
  __syncthreads();
  auto work_of = [&](int Lq, int Lk, int Lc, int mb) -> int {
    const int m0 = entry_row0(Lq, mb);
    const int n0 = sub_tile_blocks(m0, Lq, Lk, Lc, causal);
    const int n1 = sub_tile_blocks(m0 + kSubRows, Lq, Lk, Lc, causal);
    return min(kPlanBins - 1, max(n0, n1));
  };
  auto ctx_of = [&](int b) -> int { return cu_ctx != nullptr ? cu_ctx[b + 1] - cu_ctx[b] : 0; };
  for (int b = tid; b < batch; b += blockDim.x) {
    const int Lq = cu_q[b + 1] - cu_q[b];
    const int Lk = cu_k[b + 1] - cu_k[b];
    const int Lc = ctx_of(b);
    const int nmb = (Lq + kTileRows - 1) / kTileRows;
    atomicAdd(&s_total, nmb);
    for (int mb = 0; mb < nmb; ++mb) atomicAdd(&bins[work_of(Lq, Lk, Lc, mb)], 1);
  }
  __syncthreads();
  {
    // Exclusive prefix over the bins in descending work order, 4 bins a
    // thread: warp scans of the thread sums, then a scan of the warp sums.
    static_assert(kPlanBins == 4 * kPlanThreads, "4 bins per planner thread");
    __shared__ int warp_sums[kPlanThreads / 32];
    const int lane = tid & 31, wid = tid >> 5;
    int c[4], tsum = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      c[i] = bins[kPlanBins - 1 - (4 * tid + i)];
      tsum += c[i];
    }
    int incl = tsum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) warp_sums[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      const int w = warp_sums[lane];
      int wi = w;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, wi, off);
        if (lane >= off) wi += v;
      }
      warp_sums[lane] = wi - w;
    }
    __syncthreads();
    int run = warp_sums[wid] + incl - tsum;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      bins[kPlanBins - 1 - (4 * tid + i)] = run;
      run += c[i];
    }
  }
  if (tid == 0) {
    // More entries than the workspace holds means cu_seqlens_q does not end
    // at total_q: report it and compute only what fits.
    if (s_total > capacity) atomicOr(&g_mla_status, MLA_DEVSTAT_PLAN_OVERFLOW);
    const int e = min(s_total, capacity);
    ws->num_entries = e;
    ws->num_tiles = e * num_heads * nsplit;
    ws->next_tile = 0;
  }
  __syncthreads();
  for (int b = tid; b < batch; b += blockDim.x) {
    const int Lq = cu_q[b + 1] - cu_q[b];
    const int Lk = cu_k[b + 1] - cu_k[b];
    const int Lc = ctx_of(b);
    const int nmb = (Lq + kTileRows - 1) / kTileRows;
    for (int mb = nmb - 1; mb >= 0; --mb) {
      const int pos = atomicAdd(&bins[work_of(Lq, Lk, Lc, mb)], 1);
      if (pos < capacity) entries[pos] = make_int2(b, mb);
    }
  }
}

// Heads taken entry-major at the end of the list: enough for kTailRounds
// rounds of the clusters, at least one.
__device__ __forceinline__ int tail_heads(int num_heads, int num_entries, int nclusters) {
  const int want = (kTailRounds * nclusters + num_entries - 1) / max(num_entries, 1);
  return max(1, min(num_heads, want));
}

// Coordinates of tile t of the list: head-major over the sorted entries,
// then entry-major over the last `tail` heads (see the file comment); the
// splits of one (entry, head) are consecutive.
__device__ __forceinline__ TileInfo tile_info(const Params& p, int t, int num_tiles,
                                              int num_entries, int tail) {
  TileInfo ti;
  if (t < num_tiles) {
    const int split = t % p.nsplit;
    t /= p.nsplit;
    const int H = p.num_heads;
    const int bulk = (H - tail) * num_entries;
    int h, e;
    if (t < bulk) {
      h = t / num_entries;
      e = t - h * num_entries;
    } else {
      const int u = t - bulk;
      e = u / tail;
      h = H - tail + (u - e * tail);
    }
    const int2 en = p.entries[e];
    ti.q_start = p.cu_q[en.x];
    ti.Lq = p.cu_q[en.x + 1] - ti.q_start;
    ti.k_start = p.cu_k[en.x];
    ti.Lk = p.cu_k[en.x + 1] - ti.k_start;
    ti.c_start = p.cu_ctx != nullptr ? p.cu_ctx[en.x] : 0;
    ti.Lc = p.cu_ctx != nullptr ? p.cu_ctx[en.x + 1] - ti.c_start : 0;
    ti.m0 = entry_row0(ti.Lq, en.y);
    ti.hs = h | (split << 16);
  } else {
    ti.q_start = ti.Lq = ti.k_start = ti.Lk = ti.c_start = ti.Lc = ti.m0 = ti.hs = 0;
  }
  return ti;
}

// KV blocks of the tile's two sub-tiles in its split, and the split's first
// block.
__device__ __forceinline__ void tile_blocks(const TileInfo& t, int causal, int nsplit,
                                            int (&n)[2], int& lo) {
  const int f0 = sub_tile_blocks(t.m0, t.Lq, t.Lk, t.Lc, causal);
  const int f1 = sub_tile_blocks(t.m0 + kSubRows, t.Lq, t.Lk, t.Lc, causal);
  const int nmax = max(f0, f1);
  lo = split_lo(nmax, t.split(), nsplit);
  n[0] = split_count(f0, nmax, t.split(), nsplit);
  n[1] = split_count(f1, nmax, t.split(), nsplit);
}

// 32-byte store (the address must be 32-byte aligned).  A thread writes one
// output row; in 32-byte pieces each store fills whole L2 sectors, where
// 16-byte pieces leave every sector to two separate partial writes.
__device__ __forceinline__ void st_global_v8(void* addr, const uint32_t (&v)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(addr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
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

template <int DQK>
__global__ void __launch_bounds__(kThreads, 1)
    dense_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_kc,
                     const __grid_constant__ CUtensorMap tm_vc, const Params p) {
  using G = Geo<DQK>;
  constexpr int kQkChunks = G::kQkChunks;
  constexpr int kKUnits = G::kKUnits;
  constexpr int kSlots = G::kSlots;
  constexpr int kKSlotBytes = G::kKSlotBytes;
  constexpr int kQSubBytes = G::kQSubBytes;
  constexpr int kQBytes = G::kQBytes;
  constexpr int kRingBytes = G::kRingBytes;
  using BarsT = Bars<kSlots>;
  extern __shared__ uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = static_cast<int>(blockIdx.x >> 1);
  const int nclusters = static_cast<int>(gridDim.x >> 1);

  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sQ = smem_u32(base);
  const uint32_t sRingK = sQ + kQBytes;                  // kSlots x kKSlotBytes
  const uint32_t sRingV = sRingK + kSlots * kKSlotBytes;  // kSlots x 16 KB
  BarsT* bars = reinterpret_cast<BarsT*>(base + kQBytes + kRingBytes);
  volatile int* abort_flag = &bars->abort;
  // the leader CTA's copy of a barrier (cluster address)
  auto lead = [&](uint64_t* bar) -> uint32_t { return mapa_shared(smem_u32(bar), 0); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      // both producers arrive on every tile, with or without a Q load, so
      // neither can fall behind the q_empty phase it waits for
      mbar_init(smem_u32(&bars->q_full[i]), 2);
      mbar_init(smem_u32(&bars->q_empty[i]), 1);
      mbar_init(smem_u32(&bars->s_full[i]), 1);
      mbar_init(smem_u32(&bars->p_full[i]), 8);
      mbar_init(smem_u32(&bars->o_full[i]), 1);
      mbar_init(smem_u32(&bars->o_empty[i]), 8);
    }
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(smem_u32(&bars->full_kv[i]), 1);
      mbar_init(smem_u32(&bars->empty_k[i]), 1);
      mbar_init(smem_u32(&bars->empty_v[i]), 1);
    }
    for (int i = 0; i < kTileSlots; ++i) {
      mbar_init(smem_u32(&bars->tile_full[i]), 1);
      // readers of a slot: the peer's producer, the MMA warp and the 16
      // softmax warps of the pair
      mbar_init(smem_u32(&bars->tile_empty[i]), 18);
    }
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc_pair(smem_u32(&bars->tmem_base), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint64_t tlim = p.timeout_ns;
  const int causal = p.causal;
  const int num_tiles = p.ws->num_tiles;
  const int num_entries = p.ws->num_entries;
  const int tail = tail_heads(p.num_heads, num_entries * p.nsplit, nclusters);
  auto wait = [&](uint32_t bar, uint32_t parity, unsigned err) -> bool {
    return mbar_wait_cluster(bar, parity, abort_flag, err, tlim);
  };
  // Slot and phase of the k-th tile in the hand-off ring.
  auto tile_slot = [](int k) { return k % kTileSlots; };
  auto tile_par = [](int k) { return static_cast<uint32_t>(k / kTileSlots) & 1u; };

  if (warp >= 8) {
    setmaxnreg_dec<kOtherRegs>();
  if (warp == 8) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      if (p.cu_ctx != nullptr) {
        prefetch_tensormap(&tm_kc);
        prefetch_tensormap(&tm_vc);
      }
      const uint64_t pol_kv = l2_policy_evict_last();
      const uint64_t pol_q = l2_policy_evict_first();
      int blk = 0;  // KV blocks issued so far (slot = blk % kSlots)
      bool ok = true;
      for (int k = 0; ok; ++k) {
        // The leader takes the cluster's next tile and publishes it to both
        // CTAs; the peer's producer reads its copy.
        const int ts = tile_slot(k);
        TileInfo ti;
        if (leader) {
          if (!(ok = wait(smem_u32(&bars->tile_empty[ts]), tile_par(k) ^ 1u,
                          MLA_DEVSTAT_WAIT_TIMEOUT_LOAD)))
            break;
          const int t = k == 0 ? cluster : nclusters + atomicAdd(&p.ws->next_tile, 1);
          ti = tile_info(p, t, num_tiles, num_entries, tail);
          // Into both CTAs' slot: the barrier's phase completes once the
          // 32 bytes have landed (st.async counts them on it).
          const uint32_t a = smem_u32(&bars->tiles[ts]);
          for (uint32_t r = 0; r < 2; ++r) {
            const uint32_t fb = mapa_shared(smem_u32(&bars->tile_full[ts]), r);
            mbar_arrive_expect_tx_cluster(fb, static_cast<uint32_t>(sizeof(TileInfo)));
            st_async_v4(mapa_shared(a, r), ti.q_start, ti.Lq, ti.k_start, ti.Lk, fb);
            st_async_v4(mapa_shared(a + 16, r), ti.c_start, ti.Lc, ti.m0, ti.hs, fb);
          }
        } else {
          if (!(ok = wait(smem_u32(&bars->tile_full[ts]), tile_par(k),
                          MLA_DEVSTAT_WAIT_TIMEOUT_LOAD)))
            break;
          ti = bars->tiles[ts];
          if (ti.valid()) mbar_arrive_release_cluster(lead(&bars->tile_empty[ts]));
        }
        if (!ti.valid()) break;
        int nb[2], lo;
        tile_blocks(ti, causal, p.nsplit, nb, lo);
        const int h = ti.head();
        const int nblk = max(nb[0], nb[1]);
        // The tile's first K/V block goes out before its Q: its ring slot is
        // freed by MMAs three blocks back, while Q's buffers wait for the
        // previous tile's last S MMAs -- so the MMA warp, which needs block 0
        // at the previous tile's last block, does not wait for the Q reload.
        const int nctx = blocks_for(ti.Lc);  // the context's blocks come first
        auto issue_kv = [&](int n) -> bool {  // block n of the tile, the blk-th overall
          const int slot = blk % kSlots;
          const uint32_t par = (static_cast<uint32_t>(blk / kSlots) & 1u) ^ 1u;
          const int bi = lo + n;  // block of the tile's sequence
          const bool in_ctx = bi < nctx;
          const int key0 = in_ctx ? ti.c_start + bi * kBlockKeys
                                  : ti.k_start + (bi - nctx) * kBlockKeys;
          const CUtensorMap* mk = in_ctx ? &tm_kc : &tm_k;
          const CUtensorMap* mv = in_ctx ? &tm_vc : &tm_v;
          // K: this CTA's 64 keys, three 64-dim chunks of the 192
          if (!wait(smem_u32(&bars->empty_k[slot]), par, MLA_DEVSTAT_WAIT_TIMEOUT_LOAD))
            return false;
          // one barrier per block for K and V: the MMA warp waits once per block
          if (leader)
            mbar_arrive_expect_tx(smem_u32(&bars->full_kv[slot]), 2 * (kKSlotBytes + kVSlotBytes));
          const uint32_t kbar = lead(&bars->full_kv[slot]);
#pragma unroll
          for (int u = 0; u < kKUnits; ++u)
            tma_load_3d_pair(sRingK + slot * kKSlotBytes + u * kUnitBytes, mk, 64 * u, h,
                             key0 + static_cast<int>(rank) * kHalfKeys, kbar, pol_kv);
          ++blk;  // issued (its V follows on the same barrier)
          // V: all 128 keys (two units of 64), this CTA's 64 of the 128 value dims
          if (!wait(smem_u32(&bars->empty_v[slot]), par, MLA_DEVSTAT_WAIT_TIMEOUT_LOAD))
            return false;
#pragma unroll
          for (int u = 0; u < kVUnits; ++u)
            tma_load_3d_pair(sRingV + slot * kVSlotBytes + u * kUnitBytes, mv,
                             static_cast<int>(rank) * kHalfDv, h, key0 + 64 * u, kbar, pol_kv);
          return true;
        };
        if (nblk > 0) ok = issue_kv(0);
        // Q rows of this CTA, once the previous tile's last S MMA has read them.
        for (int i = 0; i < 2 && ok; ++i) {
          if (!(ok = wait(smem_u32(&bars->q_empty[i]), (static_cast<uint32_t>(k) & 1u) ^ 1u,
                          MLA_DEVSTAT_WAIT_TIMEOUT_LOAD)))
            break;
          // Both CTAs' producers arrive on the leader's q_full for every
          // tile: the MMA warp then cannot finish with a tile's Q (and
          // commit q_empty) before each producer has passed its q_empty
          // wait for that tile.  Otherwise, for a sub-tile without rows
          // (nothing to load), a late producer could find q_empty two
          // phases on and wait on the wrong phase.
          const uint32_t qbar = lead(&bars->q_full[i]);
          if (nb[i] > 0) {
            if (leader)
              mbar_arrive_expect_tx(smem_u32(&bars->q_full[i]), 2 * kQSubBytes);
            else
              mbar_arrive_cluster(qbar);
#pragma unroll
            for (int c = 0; c < kQkChunks; ++c)
              tma_load_3d_pair(sQ + (i * kQkChunks + c) * kQChunkBytes, &tm_q, 64 * c, h,
                               ti.q_start + ti.m0 + i * kSubRows + static_cast<int>(rank) * kCtaRows,
                               qbar, pol_q);
          } else {
            mbar_arrive_cluster(qbar);
          }
        }
        for (int n = 1; n < nblk && ok; ++n) ok = issue_kv(n);
      }
      if (!ok && leader) {
        // Unwinding: let the copies already issued land before the CTA exits.
        volatile int no_abort = 0;
        for (int b = max(0, blk - kSlots); b <= blk; ++b) {
          const uint32_t par = static_cast<uint32_t>(b / kSlots) & 1u;
          mbar_wait(smem_u32(&bars->full_kv[b % kSlots]), par, &no_abort, 0, tlim / 8);
        }
      }
    }
  } else if (warp == 9) {
    // -------------------------------------------- MMA issuer (leader only)
    if (leader) {
      bool ok = true;
      auto wait_bar = [&](uint32_t bar, uint32_t parity) -> bool {
        const bool r = __all_sync(0xffffffffu, wait(bar, parity, MLA_DEVSTAT_WAIT_TIMEOUT_MMA));
        tc_fence_after();
        return r;
      };
      // K and V of block b (one barrier); V(b) is covered by the wait that
      // preceded S(b).
      auto wait_kv = [&](int b) -> bool {
        return wait_bar(smem_u32(&bars->full_kv[b % kSlots]), static_cast<uint32_t>(b / kSlots) & 1u);
      };
      auto commit_both = [&](uint64_t* bar) { tc_commit_pair_elect(smem_u32(bar), 0x3); };
      // Descriptors: built once per burst, then advanced by adding to the
      // start-address field (bits 0..13, in 16-byte units); no field carries
      // since every operand lies below 256 KB of shared memory.
      auto issue_s = [&](int i, int b) {
        const uint32_t kslot = sRingK + (b % kSlots) * kKSlotBytes;
#pragma unroll 1
        for (int c = 0; c < kQkChunks; ++c) {
          // four MMAs of 16 dims (32 bytes) each
          mma2_ss_x4_elect(tmem + i * 128, sdesc_sw128(sQ + (i * kQkChunks + c) * kQChunkBytes, 16, 1024),
                           sdesc_sw128(kslot + c * kUnitBytes, 16, 1024), kIdescQK, c > 0 ? 1u : 0u);
        }
        commit_both(&bars->s_full[i]);
      };
      auto issue_pv = [&](int i, int b, bool first) {
        const uint32_t tO = tmem + 256 + i * 128;
        const uint32_t vslot = sRingV + (b % kSlots) * kVSlotBytes;
#pragma unroll 1
        for (int u = 0; u < kVUnits; ++u) {  // 64 keys per unit
          // four MMAs of 16 keys (16 rows of 128 bytes; 16 bf16 of P = 8 columns) each
          mma2_ts_x4_elect(tO, tmem + i * 128 + u * 32,
                           sdesc_sw128(vslot + u * kUnitBytes, kUnitBytes, 1024), kIdescPV,
                           (!first || u > 0) ? 1u : 0u);
        }
      };

      int blk = 0;            // first KV block (global count) of the current tile
      int p_cnt[2] = {0, 0};  // P blocks consumed per sub-tile (p_full parity)
      int o_cnt[2] = {0, 0};  // O-using tiles per sub-tile (o_full / o_empty parity)
      // First S MMAs of a tile when the previous tile did not issue them.
      auto start_tile = [&](const int (&n)[2], int b, int k) -> bool {
        for (int i = 0; i < 2; ++i)
          if (!wait_bar(smem_u32(&bars->q_full[i]), static_cast<uint32_t>(k) & 1u)) return false;
        if (max(n[0], n[1]) > 0) {
          if (!wait_kv(b)) return false;
          for (int i = 0; i < 2; ++i) {
            if (n[i] > 0) issue_s(i, b);
            if (n[i] <= 1) commit_both(&bars->q_empty[i]);
          }
          commit_both(&bars->empty_k[b % kSlots]);
        } else {
          for (int i = 0; i < 2; ++i) commit_both(&bars->q_empty[i]);
        }
        return true;
      };

      // Tile k from the hand-off ring: whether it exists and the KV blocks
      // of its two sub-tiles (read by every lane; lane 0 frees the slot).
      auto fetch = [&](int k, int& valid, int (&n)[2]) -> bool {
        const int ts = tile_slot(k);
        if (!wait_bar(smem_u32(&bars->tile_full[ts]), tile_par(k))) return false;
        const TileInfo ti = bars->tiles[ts];
        valid = ti.valid();
        int lo;
        tile_blocks(ti, causal, p.nsplit, n, lo);
        __syncwarp();
        if (valid && lane == 0) mbar_arrive(smem_u32(&bars->tile_empty[ts]));
        return true;
      };

      int k = 0;
      int cur_valid = 0, nxt_valid = 0;
      int nb[2] = {0, 0}, nbn[2] = {0, 0};
      ok = fetch(k, cur_valid, nb);
      if (ok && cur_valid) ok = start_tile(nb, blk, k);
      while (ok && cur_valid) {
        const int nblk = max(nb[0], nb[1]);
        // The next tile is read when it is first needed (the last block of
        // this one): the producer publishes it only after it has issued
        // this tile's loads.
        if (nblk == 0 && !(ok = fetch(k + 1, nxt_valid, nbn))) break;
        for (int n = 0; n < nblk && ok; ++n) {
          const int b = blk + n;  // this KV block; the next one is b + 1
          const bool last = n + 1 == nblk;
          if (last && !(ok = fetch(k + 1, nxt_valid, nbn))) break;
          bool next_s[2] = {n + 1 < nb[0], n + 1 < nb[1]};
          if (last) {
            next_s[0] = nbn[0] > 0;
            next_s[1] = nbn[1] > 0;
          }
          const bool more = next_s[0] || next_s[1];
          if (more && !(ok = wait_kv(b + 1))) break;
          for (int i = 0; i < 2 && ok; ++i) {
            if (n < nb[i]) {
              if (n == 0 && !(ok = wait_bar(smem_u32(&bars->o_empty[i]),
                                            (static_cast<uint32_t>(o_cnt[i]) & 1u) ^ 1u)))
                break;
              if (!(ok = wait_bar(smem_u32(&bars->p_full[i]),
                                  static_cast<uint32_t>(p_cnt[i]) & 1u)))
                break;
              ++p_cnt[i];
              issue_pv(i, b, n == 0);
              if (n == nb[i] - 1) {
                commit_both(&bars->o_full[i]);
                ++o_cnt[i];
              }
            }
            if (i == 1) commit_both(&bars->empty_v[b % kSlots]);  // V(b) no longer needed
            if (last && nxt_valid &&
                !(ok = wait_bar(smem_u32(&bars->q_full[i]), static_cast<uint32_t>(k + 1) & 1u)))
              break;
            if (next_s[i]) {
              issue_s(i, b + 1);
              // Q_i is free after the last S MMA of its tile
              const int nbi = last ? nbn[i] : nb[i];
              const int nidx = last ? 0 : n + 1;
              if (nidx == nbi - 1) commit_both(&bars->q_empty[i]);
            } else if (last && nxt_valid) {
              commit_both(&bars->q_empty[i]);  // no S for it in the next tile
            }
          }
          if (ok && more) commit_both(&bars->empty_k[(b + 1) % kSlots]);  // K(b+1) read by both S
        }
        if (!ok) break;
        if (nblk == 0 && nxt_valid && !(ok = start_tile(nbn, blk, k + 1))) break;
        blk += nblk;
        ++k;
        cur_valid = nxt_valid;
        nb[0] = nbn[0];
        nb[1] = nbn[1];
      }
      // Wait until every MMA issued above has completed.
      tc_commit_pair_elect(smem_u32(&bars->drain), 0x1);
      __syncwarp();
      volatile int no_abort = 0;
      mbar_wait_cluster(smem_u32(&bars->drain), 0, &no_abort, MLA_DEVSTAT_WAIT_TIMEOUT_MMA, tlim);
    }
  }
  } else {
    setmaxnreg_inc<kSoftmaxRegs>();
    // ------------------------------------------------ softmax warpgroups
    const int sub = warp >> 2;
    const int wq = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + sub * 128;
    const uint32_t tO = tmem + lane_off + 256 + sub * 128;
    const float sl2 = p.scale_log2;
    const uint64_t c2 = pack_f32x2(sl2, sl2);
    const Exp2PolyConsts pk2 = exp2_poly_consts();
    const uint32_t sbar = smem_u32(&bars->s_full[sub]);
    const uint32_t pbar_lead = lead(&bars->p_full[sub]);
    const uint32_t obar_lead = lead(&bars->o_empty[sub]);
    int s_cnt = 0;  // S blocks consumed (s_full parity)
    int o_cnt = 0;  // O-using tiles (o_full parity)
    bool ok = true;
    // The second half of the previous tile's output row (64 bf16 as 32
    // words), stored once the next tile's first P is published: the stores
    // of a tile's epilogue otherwise delay that P, on which the MMA warp
    // waits at the tile boundary (32-byte-aligned bf16 outputs only).
    uint32_t dfr[32];
    __nv_bfloat16* dfr_row = nullptr;
    auto flush_dfr = [&]() {
      if (dfr_row != nullptr) {
#pragma unroll
        for (int v8 = 0; v8 < 4; ++v8)
          st_global_v8(dfr_row + 64 + 16 * v8, *reinterpret_cast<const uint32_t(*)[8]>(&dfr[8 * v8]));
        dfr_row = nullptr;
      }
    };
    for (int k = 0; ok; ++k) {
      const int ts = tile_slot(k);
      ok = __all_sync(0xffffffffu, wait(smem_u32(&bars->tile_full[ts]), tile_par(k),
                                        MLA_DEVSTAT_WAIT_TIMEOUT_SOFTMAX));
      if (!ok) break;
      // The block loop needs only the row and key limits; the epilogue reads
      // the tile's coordinates from the slot again (it stays valid until
      // this warp frees it), which keeps them out of registers meanwhile.
      const TileInfo* slot = &bars->tiles[ts];
      if (!slot->valid()) break;
      const int Lk = slot->Lk;
      const int Lc = slot->Lc;
      const int nc = blocks_for(Lc);  // context blocks (every context key is visible)
      // first row of this CTA's part of the sub-tile, and the last own key
      // that row sees (bottom-right causal: row i sees keys j <= i + Lk - Lq)
      const int row0 = slot->m0 + sub * kSubRows + static_cast<int>(rank) * kCtaRows;
      const int diag = row0 + Lk - slot->Lq;
      int nb, lo;  // this sub-tile's blocks in the tile's split, from block lo on
      {
        int n2[2];
        tile_blocks(*slot, causal, p.nsplit, n2, lo);
        nb = n2[sub];
      }
      const int ldiag = diag + wq * 32 + lane;  // this thread's row's last key
      const int lim = causal ? min(Lk, ldiag + 1) : Lk;  // own keys [0, lim) visible
      float m_run = -INFINITY;  // running max of scale*log2(e)*s (lazily updated)
      float l_run = 0.f;        // running sum of the fp32 weights exp2(scaled s - m_run)

      for (int n = 0; n < nb; ++n) {
        ok = __all_sync(0xffffffffu, wait(sbar, static_cast<uint32_t>(s_cnt) & 1u,
                                          MLA_DEVSTAT_WAIT_TIMEOUT_SOFTMAX));
        if (!ok) break;
        ++s_cnt;
        tc_fence_after();
        uint32_t sraw[128];
        tmem_ld_x128_wait(tS, sraw);
        float x[128];
#pragma unroll
        for (int j = 0; j < 128; ++j) x[j] = __uint_as_float(sraw[j]);
        // Blocks [0, nc) hold context keys 128 n + j, visible below Lc; the
        // sequence's own keys follow, visible below the row's limit.  A block
        // that every row of the CTA sees whole needs no mask.
        const int bi = lo + n;  // block of the tile's sequence
        const bool in_ctx = bi < nc;
        const int kbase = (in_ctx ? bi : bi - nc) * kBlockKeys;
        const bool full_blk =
            in_ctx ? kbase + kBlockKeys <= Lc
                   : (kbase + kBlockKeys <= Lk) && (!causal || kbase + kBlockKeys - 1 <= diag);
        if (!full_blk) {
          const int klim = in_ctx ? Lc : lim;
#pragma unroll
          for (int j = 0; j < 128; ++j)
            if (kbase + j >= klim) x[j] = -INFINITY;
        }
        float m8[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) m8[t] = x[t];
#pragma unroll
        for (int j = 8; j < 120; j += 16)
#pragma unroll
          for (int t = 0; t < 8; ++t) m8[t] = fmax3(m8[t], x[j + t], x[j + 8 + t]);
#pragma unroll
        for (int t = 0; t < 8; ++t) m8[t] = fmaxf(m8[t], x[120 + t]);
        const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                               fmaxf(m8[6], m8[7]));
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
        const uint64_t negm2 = pack_f32x2(-m_use, -m_use);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // 32 scores -> 16 packed bf16 pairs per store
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            // 14 of every 16 pairs on the MUFU unit, 2 on the FMA pipe
            if ((j & 7) < 7)
              pk[j] = softmax_pair_mufu(x[32 * c + 2 * j], x[32 * c + 2 * j + 1], c2, negm2,
                                        acc[j & 3]);
            else
              pk[j] = softmax_pair_poly(x[32 * c + 2 * j], x[32 * c + 2 * j + 1], c2, negm2, pk2,
                                        acc[j & 3]);
          }
          tmem_st_x16(tS + 16u * c, pk);
        }
        l_run += (sum_f32x2(acc[0]) + sum_f32x2(acc[1])) + (sum_f32x2(acc[2]) + sum_f32x2(acc[3]));
        // O(n-1) is complete (its MMAs precede S(n) in issue order) and PV(n)
        // waits for p_full, so O can be rescaled here, after the scores died.
        if (n > 0 && __any_sync(0xffffffffu, need)) rescale_o_row(tO, alpha);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(pbar_lead);
        if (n == 0) flush_dfr();
      }
      if (!ok) break;
      const int e_lq = bars->tiles[ts].Lq;
      const int e_q0 = bars->tiles[ts].q_start;
      const int e_h = bars->tiles[ts].head();
      const int e_split = bars->tiles[ts].split();
      const int r = bars->tiles[ts].m0 + sub * kSubRows + static_cast<int>(rank) * kCtaRows +
                    wq * 32 + lane;  // this thread's row within the sequence
      // Done with the tile's ring slot.  Freed here rather than at the start
      // of the tile so that the cluster-scope release does not wait for the
      // previous epilogue's stores.
      __syncwarp();
      if (lane == 0) mbar_arrive_release_cluster(lead(&bars->tile_empty[ts]));

      flush_dfr();  // a tile without blocks for this sub-tile came in between
      // ------------------------------------------------------- epilogue
      // Denominator Z = l 2^m (+ 2^s for the head's sink s, in the same log2
      // units); O = O_acc 2^m / Z, LSE = log2(Z) ln 2.  Without a sink this
      // is O_acc / l and m + log2 l.  A row that saw no key keeps m_run =
      // -inf (its weights are only the tiny clamped values of the polynomial
      // path): output 0, LSE -inf, or the sink's logit.
      const bool row_ok = r >= 0 && r < e_lq;
      const size_t row_index = static_cast<size_t>(e_q0 + r) * p.num_heads + e_h;
      const size_t out_off = static_cast<size_t>(e_q0 + r) * p.out_rs +
                             static_cast<size_t>(e_h) * p.out_hs;  // first element of the row
      const bool fp8 = p.out_scale != nullptr;
      const float sink2 = p.sinks != nullptr ? p.sinks[e_h] * 1.4426950408889634f : -INFINITY;
      float lse2 = sink2;  // log2 of the row's denominator
      if (nb > 0) {
        ok = __all_sync(0xffffffffu, wait(smem_u32(&bars->o_full[sub]),
                                          static_cast<uint32_t>(o_cnt) & 1u,
                                          MLA_DEVSTAT_WAIT_TIMEOUT_SOFTMAX));
        if (!ok) break;
        tc_fence_after();
        uint32_t o[128];
        tmem_ld_x128_wait(tO, o);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(obar_lead);  // O may be overwritten now
        ++o_cnt;
        float scale_o = 0.0f;  // multiplier of O's accumulator
        if (m_run != -INFINITY) {
          if (p.sinks == nullptr) {
            scale_o = 1.0f / l_run;
            lse2 = m_run + lg2_approx(l_run);
          } else {
            const float mz = fmaxf(m_run, sink2);
            const float z = l_run * ex2_approx(m_run - mz) + ex2_approx(sink2 - mz);
            scale_o = ex2_approx(m_run - mz) / z;
            lse2 = mz + lg2_approx(z);
          }
        }
        if (row_ok && p.nsplit > 1) {
          // split-KV: this split's O (normalised by its own sum) in fp32
          float* prow =
              p.o_part + (static_cast<size_t>(e_split) * p.total_q * p.num_heads + row_index) * kDv;
          if (p.wide_out & 2) {
#pragma unroll
            for (int v8 = 0; v8 < 16; ++v8) {
              uint32_t w[8];
#pragma unroll
              for (int j = 0; j < 8; ++j)
                w[j] = __float_as_uint(__uint_as_float(o[8 * v8 + j]) * scale_o);
              st_global_v8(prow + 8 * v8, w);
            }
          } else {
            float4* prow4 = reinterpret_cast<float4*>(prow);
#pragma unroll
            for (int v4 = 0; v4 < 32; ++v4)
              prow4[v4] = make_float4(__uint_as_float(o[4 * v4]) * scale_o,
                                      __uint_as_float(o[4 * v4 + 1]) * scale_o,
                                      __uint_as_float(o[4 * v4 + 2]) * scale_o,
                                      __uint_as_float(o[4 * v4 + 3]) * scale_o);
          }
        } else if (row_ok && !fp8) {
          __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + out_off;
          if (p.wide_out & 1) {
#pragma unroll
            for (int v8 = 0; v8 < 4; ++v8) {  // 16 bf16 per store
              uint32_t pk[8];
#pragma unroll
              for (int j = 0; j < 8; ++j)
                pk[j] = pack_bf16x2(__uint_as_float(o[16 * v8 + 2 * j]) * scale_o,
                                    __uint_as_float(o[16 * v8 + 2 * j + 1]) * scale_o);
              st_global_v8(orow + 16 * v8, pk);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j)
              dfr[j] = pack_bf16x2(__uint_as_float(o[64 + 2 * j]) * scale_o,
                                   __uint_as_float(o[64 + 2 * j + 1]) * scale_o);
            dfr_row = orow;
          } else {
            uint4* orow4 = reinterpret_cast<uint4*>(orow);
#pragma unroll
            for (int v4 = 0; v4 < 16; ++v4) {
              uint32_t pk[4];
#pragma unroll
              for (int j = 0; j < 4; ++j)
                pk[j] = pack_bf16x2(__uint_as_float(o[8 * v4 + 2 * j]) * scale_o,
                                    __uint_as_float(o[8 * v4 + 2 * j + 1]) * scale_o);
              orow4[v4] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
          }
        } else if (row_ok) {
          // e4m3 of O / out_scale: round to nearest even, saturated at 448
          const float qs = scale_o / *p.out_scale;
          uint8_t* orow = static_cast<uint8_t*>(p.out) + out_off;
          if (p.wide_out & 1) {
#pragma unroll
            for (int v32 = 0; v32 < 4; ++v32) {  // 32 e4m3 per store
              uint32_t pk[8];
#pragma unroll
              for (int j = 0; j < 8; ++j)
                pk[j] = pack_e4m3x4(__uint_as_float(o[32 * v32 + 4 * j]) * qs,
                                    __uint_as_float(o[32 * v32 + 4 * j + 1]) * qs,
                                    __uint_as_float(o[32 * v32 + 4 * j + 2]) * qs,
                                    __uint_as_float(o[32 * v32 + 4 * j + 3]) * qs);
              st_global_v8(orow + 32 * v32, pk);
            }
          } else {
            uint4* orow4 = reinterpret_cast<uint4*>(orow);
#pragma unroll
            for (int v16 = 0; v16 < 8; ++v16) {
              uint32_t pk[4];
#pragma unroll
              for (int j = 0; j < 4; ++j)
                pk[j] = pack_e4m3x4(__uint_as_float(o[16 * v16 + 4 * j]) * qs,
                                    __uint_as_float(o[16 * v16 + 4 * j + 1]) * qs,
                                    __uint_as_float(o[16 * v16 + 4 * j + 2]) * qs,
                                    __uint_as_float(o[16 * v16 + 4 * j + 3]) * qs);
              orow4[v16] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
          }
        }
      } else if (row_ok && p.nsplit > 1) {
        // no key of this split: a zero partial with LSE -inf
        float4* prow = reinterpret_cast<float4*>(
            p.o_part + (static_cast<size_t>(e_split) * p.total_q * p.num_heads + row_index) * kDv);
        for (int v = 0; v < 32; ++v) prow[v] = make_float4(0.f, 0.f, 0.f, 0.f);
      } else if (row_ok) {
        // no visible key: zeros (bf16 rows of 256 bytes, e4m3 rows of 128)
        uint4* orow = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) +
                                               out_off * (fp8 ? 1 : 2));
        const int n16 = fp8 ? 8 : 16;
        for (int v = 0; v < n16; ++v) orow[v] = make_uint4(0u, 0u, 0u, 0u);
      }
      if (row_ok && p.nsplit > 1)
        p.lse_part[(static_cast<size_t>(e_split) * p.num_heads + e_h) * p.total_q + e_q0 + r] =
            lse2 * 0.69314718055994530942f;
      else if (row_ok && p.lse != nullptr)
        p.lse[static_cast<size_t>(e_h) * p.total_q + e_q0 + r] = lse2 * 0.69314718055994530942f;
    }
    flush_dfr();  // the last tile's deferred half
  }

  // Neither CTA leaves (or frees TMEM) while the pair's MMAs may still
  // read its shared memory or write its TMEM.
  tc_fence_before();
  cluster_sync();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace dense
}  // namespace mla
