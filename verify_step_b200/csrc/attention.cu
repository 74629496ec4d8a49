// Verify attention and drafter cross-attention over a paged KV cache (sm_100a).
//
// What is computed: "Gemma 4 MTP: drafter drafts, target verifies", section "drafter internal
// architecture" (k+1 positions verified in one pass; each drafter layer attends directly into
// the target's KV cache).  Query j of sequence b sits at t = L_b + j (verify) or q_pos[b]
// (drafter) and attends to keys p in [lo, hi]: lo = max(0, t - window + 1) on a sliding layer,
// 0 on a global one; hi = t (verify) or min(t, L_b - 1) (drafter).  Query head h reads kv head
// h / G.
//
// bf16 design (decode attention is bandwidth-bound: GeekNews summary of the Google blog,
// section "why speculative decoding"):
//  * Persistent CTAs split the flattened list of (sequence, kv head, 16-key tile) work evenly
//    (stream-K): every CTA streams the same number of KV bytes however ragged the contexts.
//  * A producer warp moves each 16-key K and V tile of one kv head (contiguous in the
//    [num_blocks, h_kv, block_size, D] layout) into shared memory once, by TMA
//    (cp.async.bulk.tensor, 128-byte swizzle, no multicast), through an mbarrier ring.
//  * The tile is reused by every query row of the item: the G query heads of the kv head times
//    the n_q verify positions (M = G * n_q rows, up to 24 per CTA in 8-row blocks; larger items
//    take groups of CTAs streaming the same tiles).
//  * Compute warps own a D slice of 128 columns.  Keys are the M side of the bf16 mma.sync
//    tensor-core products (S^T = K Q^T, O^T += V^T P^T, float32 accumulation) and query rows
//    the N side, so few rows cost little padding.  S^T partials over the slices are summed
//    through shared memory (fixed order, so every warp gets the same scores); the online
//    softmax runs in registers, masking only the tiles at a row's range ends and rescaling only
//    when a row maximum grows by more than 2^8.
//  * Items split across CTAs leave (m, l, o) partials in the workspace; a combine kernel merges
//    them in CTA order (deterministic).  Items one CTA finishes are written directly.
//
// float32 path: one warp per query row, plain FMA (the tiny float32 configuration).
#include <algorithm>
#include <cfloat>

#include "common.cuh"
#include "host.cuh"

namespace sdv {
namespace attn {

constexpr int kTile = 16;
constexpr float kRescale = 8.f;  // log2 headroom of the lazily rescaled softmax
constexpr int kMaxGroups = 1024;  // stream-K groups of the split-KV grid at most

struct Params {
  int B, n_q, Hq, Hkv, G, D, bs, mbps, num_blocks, window, M;
  int Mpad;          // rows of a workspace slot (split-KV kernel)
  int is_draft;
  int q_offset;      // query position ctx_len[b] + q_offset when q_pos is null
  float scale_log2;  // scale * log2(e)
  float scale;
  const void *q;
  const int32_t *table;
  const int32_t *ctx_len;
  const int32_t *q_pos;
  void *out;
  float *ws_o;   // [slots][Mpad][D]
  float *ws_ml;  // [slots][Mpad][2]
  // Verify on the cluster (sliding-window) kernel with one 16-row query tile: the new rows
  // come from k_new / v_new, and the kernel also writes them into the cache.  Null when a
  // separate append kernel ran first (or for the drafter).
  const void *k_new;
  const void *v_new;
  void *k_cache;
  void *v_cache;
  int kv3d;        // the K / V tensor maps are the 3D chunk view (one box per tile)
  int P;           // CTA groups of the persistent split-KV grid (stream-K units)
  int row_groups;  // CTAs per group: each takes one row group of the item, same tile range
  int *status;
};

// Keys an item (sequence b, any kv head) reads: tiles [tf, tf + n) of 16 positions, with
// lo_min / hi_max the union of the rows' key ranges.
struct SeqRange {
  int L, tf, n, lo_min, hi_max;
};

__device__ __forceinline__ int draft_qpos(const Params &p, int b) {
  return p.q_pos != nullptr ? p.q_pos[b] : p.ctx_len[b] + p.q_offset;
}

__device__ __forceinline__ SeqRange seq_range(const Params &p, int b, bool report) {
  SeqRange r;
  r.L = p.ctx_len[b];
  r.tf = 0;
  r.n = 0;
  r.lo_min = 0;
  r.hi_max = -1;
  int lo, hi;
  if (!p.is_draft) {
    if (r.L < 0) {
      if (report) record_status(p.status, SD_ERR_DEVICE);
      return r;
    }
    hi = r.L + p.n_q - 1;
    lo = p.window > 0 ? max(0, r.L - p.window + 1) : 0;
  } else {
    const int qp = draft_qpos(p, b);
    if (r.L < 0 || qp < 0) {
      if (report) record_status(p.status, SD_ERR_DEVICE);
      return r;
    }
    hi = min(qp, r.L - 1);
    lo = p.window > 0 ? max(0, qp - p.window + 1) : 0;
  }
  if (hi < lo) return r;
  if (hi >= p.mbps * p.bs) {  // positions beyond the block table
    if (report) record_status(p.status, SD_ERR_DEVICE);
    return r;
  }
  r.tf = lo / kTile;
  r.n = hi / kTile - r.tf + 1;
  r.lo_min = lo;
  r.hi_max = hi;
  return r;
}

// Key range of query row `row` (row = j * G + hh) of sequence b.
__device__ __forceinline__ void row_range(const Params &p, const SeqRange &s, int b, int row,
                                          int &lo, int &hi) {
  if (row >= p.M || s.n == 0) {
    lo = 1;
    hi = 0;
    return;
  }
  if (!p.is_draft) {
    const int t = s.L + row / p.G;
    hi = t;
    lo = p.window > 0 ? max(0, t - p.window + 1) : 0;
  } else {
    const int t = draft_qpos(p, b);
    hi = min(t, s.L - 1);
    lo = p.window > 0 ? max(0, t - p.window + 1) : 0;
  }
}

// Per-sequence ranges cached in shared memory for batches up to kTabB (built once per CTA by
// one warp); larger batches recompute them from global memory.
constexpr int kTabB = 64;

struct SeqTab {
  SeqRange r[kTabB];
  long long pre[kTabB + 1];  // pre[b] = tiles of sequences before b (times h_kv)
  int ok;
};

__device__ __forceinline__ void build_tab(const Params &p, SeqTab *t) {
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  if (p.B > kTabB) {
    if (lane == 0) t->ok = 0;
    return;
  }
  long long carry = 0;
  for (int base = 0; base < p.B; base += 32) {
    const int b = base + lane;
    long long v = 0;
    if (b < p.B) {
      t->r[b] = seq_range(p, b, false);
      v = (long long)p.Hkv * t->r[b].n;
    }
    for (int o = 1; o < 32; o <<= 1) {
      const long long u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (b < p.B) t->pre[b + 1] = carry + v;
    carry += __shfl_sync(0xffffffffu, v, 31);
  }
  if (lane == 0) {
    t->pre[0] = 0;
    t->ok = 1;
  }
}

__device__ __forceinline__ SeqRange tab_range(const Params &p, const SeqTab *t, int b) {
  return t->ok ? t->r[b] : seq_range(p, b, false);
}

__device__ __forceinline__ long long total_tiles(const Params &p, const SeqTab *t) {
  if (t->ok) return t->pre[p.B];
  long long T = 0;
  for (int b = 0; b < p.B; ++b) T += (long long)p.Hkv * seq_range(p, b, false).n;
  return T;
}

// Cursor over the flattened (b, g, tile) list of one CTA.
struct Cursor {
  int b, g, tau;         // current item and tile index inside it
  SeqRange s;            // range of sequence b
  long long left;        // tiles still to process by this CTA
};

__device__ __forceinline__ void cursor_begin(const Params &p, const SeqTab *t, long long start,
                                             long long count, Cursor &c) {
  c.left = count;
  long long pre = 0;
  c.b = 0;
  c.g = 0;
  c.tau = 0;
  c.s = tab_range(p, t, 0);
  if (count <= 0) return;
  for (int b = 0; b < p.B; ++b) {
    SeqRange s = tab_range(p, t, b);
    const long long len = (long long)p.Hkv * s.n;
    if (start < pre + len) {
      c.b = b;
      c.s = s;
      const long long off = start - pre;
      c.g = (int)(off / s.n);
      c.tau = (int)(off % s.n);
      return;
    }
    pre += len;
  }
  c.left = 0;
}

// Advances to the next item after the current one finished (tau == n).
__device__ __forceinline__ void cursor_next_item(const Params &p, const SeqTab *t, Cursor &c) {
  c.tau = 0;
  if (++c.g < p.Hkv) return;
  c.g = 0;
  for (int b = c.b + 1; b < p.B; ++b) {
    SeqRange s = tab_range(p, t, b);
    if (s.n > 0) {
      c.b = b;
      c.s = s;
      return;
    }
  }
  c.left = 0;
}

// Byte offset of element (row, col) inside a [16 rows x D] bf16 tile stored as D/64 chunks of
// [16 rows x 128 B] with the 128-byte swizzle (16-byte unit u of row r stored at u ^ (r & 7)).
__device__ __forceinline__ uint32_t swz(int row, int col) {
  const int chunk = col >> 6;
  const int unit = (col >> 3) & 7;
  return (uint32_t)(chunk * (kTile * 128) + row * 128 + ((unit ^ (row & 7)) << 4) +
                    ((col & 7) << 1));
}

// Verify with the fused append: the staged tile at positions [p0, p0 + 16) of sequence b may
// hold some of the n_q new rows (positions L .. L + n_q - 1), which the cache does not have
// yet.  The calling warp, sole owner of columns [col0, col0 + DS) of the tile, copies its slice
// of those rows from k_new / v_new into the staged K and V tiles and into the cache.  Returns
// whether it wrote shared memory (the stage then needs a proxy fence before TMA reuses it).
template <int D, int DS>
__device__ __forceinline__ bool patch_new_rows(const Params &p, int b, int g, int L, int p0,
                                               int col0, uint8_t *ktile, uint8_t *vtile,
                                               int lane) {
  const int r_lo = max(L, p0) - p0, r_hi = min(L + p.n_q, p0 + kTile) - p0;
  if (r_lo >= r_hi) return false;
  constexpr int U = DS / 8;  // 16-byte units of one row's slice
  const int n = (r_hi - r_lo) * 2 * U;
  // all 16-byte pieces in flight at once (cp.async: no registers held), then from shared
  // memory into the cache
  for (int i = lane; i < n; i += 32) {
    const int r = r_lo + i / (2 * U), kv = (i / U) & 1, u = i % U;
    const __nv_bfloat16 *src = reinterpret_cast<const __nv_bfloat16 *>(kv == 0 ? p.k_new : p.v_new);
    const __nv_bfloat16 *gp = src + (((size_t)b * p.n_q + (p0 + r - L)) * p.Hkv + g) * D + col0 + u * 8;
    cp_async_16(smem_u32((kv == 0 ? ktile : vtile) + swz(r, col0 + u * 8)), gp);
  }
  cp_async_wait_all();
  __syncwarp();
  const int blk = p.table[(size_t)b * p.mbps + p0 / p.bs];  // the producer checked it
  for (int i = lane; i < n; i += 32) {
    const int r = r_lo + i / (2 * U), kv = (i / U) & 1, u = i % U;
    const int col = col0 + u * 8, t = p0 + r;
    const uint4 v = *reinterpret_cast<const uint4 *>((kv == 0 ? ktile : vtile) + swz(r, col));
    __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(kv == 0 ? p.k_cache : p.v_cache);
    *reinterpret_cast<uint4 *>(dst + (((size_t)blk * p.Hkv + g) * p.bs + (t % p.bs)) * D + col) =
        v;
  }
  return true;
}

// Split-KV tile shape: query rows are the MMA's N dimension in blocks of 8 (NB blocks per CTA),
// keys its M dimension (one 16-key tile), so an item of up to 24 rows (k + 1 = 6 positions at
// G = 4) is one CTA's work and needs no padding beyond the next multiple of 8.
template <int D, int NB, int STAGES, bool SPLIT>
struct Cfg {
  static constexpr int DS = D >= 128 ? 128 : 64;
  static constexpr int NDG = D / DS;  // compute warps, one D slice each
  static constexpr int NCW = NDG;
  // Two or three row blocks at D 512 need more registers per compute thread than 10 warps per SM
  // leave (168): the CTA is then two warpgroups, the copy warp's group handing registers to the
  // four compute warps (setmaxnreg: 4 x 32 x kRegCopy + 4 x 32 x kRegMath = 256 threads x 128
  // registers at launch, checked on the host before the first launch).
  static constexpr bool WS = SPLIT;
  static constexpr int THREADS = WS ? 256 : 32 * (NCW + 1);
  static constexpr int COPY_WARP = WS ? 0 : NCW;   // the warp issuing the tile copies
  static constexpr int MATH_WARP0 = WS ? 4 : 0;    // first compute warp
  static constexpr int kRegLaunch = 128, kRegCopy = 24, kRegMath = 232;
  static_assert(!WS || 128 * kRegCopy + 128 * kRegMath == THREADS * kRegLaunch,
                "register split must equal the launch total");
  static constexpr int ROWS = 8 * NB;
  static constexpr int TILE_BYTES = kTile * D * 2;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int RED_FLOATS = NDG > 1 ? 2 * NCW * 32 * 4 * NB : 4;
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + RED_FLOATS * 4 +
                                 16 * STAGES + 16 + 4 * (1 + STAGES) + 64 + sizeof(SeqTab) + 16;
  // two independent tile pipelines per SM (one CTA's per-tile chain of waits, MMAs and the
  // cross-warp score exchange is latency-bound on its own)
  static constexpr int MIN_CTAS = 2;
};

// Rows per CTA group for an item of M query rows: groups of at most 24 rows (three 8-row
// blocks), R groups of NB blocks each.  At D 512 groups of two or three blocks take the
// warpgroup register split (28 rows, two groups of two blocks: 271 against 290 us without).
struct RowSplit {
  int R, NB;
  bool split;
};
__host__ __device__ inline RowSplit row_split(int M, int D) {
  RowSplit s;
  s.R = (M + 23) / 24;
  const int per = (M + s.R - 1) / s.R;
  s.NB = (per + 7) / 8;
  s.split = D == 512 && s.NB >= 2;
  return s;
}

template <int D, int NB, int STAGES, bool SPLIT>
__global__ void __launch_bounds__(Cfg<D, NB, STAGES, SPLIT>::THREADS,
                                  Cfg<D, NB, STAGES, SPLIT>::MIN_CTAS)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap, const Params p) {
  using C = Cfg<D, NB, STAGES, SPLIT>;
  constexpr int DS = C::DS, NDG = C::NDG, NCW = C::NCW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *stages = smem;
  float *red = reinterpret_cast<float *>(smem + (size_t)STAGES * C::STAGE_BYTES);
  uint64_t *full = reinterpret_cast<uint64_t *>(red + C::RED_FLOATS);
  uint64_t *empty = full + STAGES;
  uint64_t *red_bar = empty + STAGES;  // [2]: partial scores of a tile are in red[buf]
  volatile int *abort_flag = reinterpret_cast<volatile int *>(red_bar + 2);
  volatile int *bad = abort_flag + 1;
  SeqTab *tab = reinterpret_cast<SeqTab *>(
      (reinterpret_cast<uintptr_t>(bad + STAGES) + 15) & ~uintptr_t(15));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW * 32);
      bad[s] = 0;
    }
    mbar_init(&red_bar[0], NCW * 32);
    mbar_init(&red_bar[1], NCW * 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  pdl_trigger();
  pdl_wait();  // everything below reads memory earlier kernels may have written
  build_tab(p, tab);
  __syncthreads();

  const long long T = total_tiles(p, tab);
  // CTAs come in groups of row_groups that stream the same tile range, one row group each
  // (the group's repeated reads of a tile are served by L2)
  const int grp = blockIdx.x / p.row_groups, rg = blockIdx.x % p.row_groups;
  const long long start = T * grp / p.P;
  const long long end = T * (grp + 1) / p.P;

  if constexpr (C::WS) {
    if (warp < 4) {
      setmaxnreg_dec<C::kRegCopy>();
      if (warp != C::COPY_WARP) return;
    } else {
      setmaxnreg_inc<C::kRegMath>();
    }
  }
  if (warp == C::COPY_WARP) {
    // ------------------------------------------------------------------- producer warp
    // The whole warp walks the cursor; its lanes fetch the block-table entries of the next 32
    // tiles of the current sequence at once (off the per-tile path), lane 0 issues the copies.
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
    }
    Cursor c;
    cursor_begin(p, tab, start, end - start, c);
    uint32_t it = 0;
    int pf_b = -1, pf_base = 0, blk_l = -1;
    while (c.left > 0) {
      const int ti = c.s.tf + c.tau;  // tile index inside sequence c.b
      if (c.b != pf_b || ti < pf_base || ti >= pf_base + 32) {
        pf_b = c.b;
        pf_base = ti;
        blk_l = -1;
        const int bidx = (ti + lane) * kTile / p.bs;
        if (ti + lane < c.s.tf + c.s.n && bidx < p.mbps)
          blk_l = p.table[(size_t)c.b * p.mbps + bidx];
      }
      const int blk = __shfl_sync(0xffffffffu, blk_l, ti - pf_base);
      int go = 1;
      if (lane == 0) {
        const int stage = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait(&empty[stage], ph ^ 1, abort_flag)) {
          record_status(p.status, SD_ERR_TIMEOUT);
          *abort_flag = 1;
          go = 0;
        } else if (blk < 0 || blk >= p.num_blocks) {
          record_status(p.status, SD_ERR_DEVICE);
          bad[stage] = 1;
          mbar_arrive(&full[stage]);
        } else {
          bad[stage] = 0;
          const int p0 = ti * kTile;
          const int row = (blk * p.Hkv + c.g) * p.bs + (p0 % p.bs);
          uint8_t *kd = stages + (size_t)stage * C::STAGE_BYTES;
          uint8_t *vd = kd + C::TILE_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          if (p.kv3d) {  // one box per tile brings every column chunk
            tma_load_3d(kd, &kmap, &full[stage], 0, row, 0);
            tma_load_3d(vd, &vmap, &full[stage], 0, row, 0);
          } else {
#pragma unroll
            for (int ch = 0; ch < D / 64; ++ch) {
              tma_load_2d(kd + ch * (kTile * 128), &kmap, &full[stage], ch * 64, row);
              tma_load_2d(vd + ch * (kTile * 128), &vmap, &full[stage], ch * 64, row);
            }
          }
        }
      }
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      ++it;
      --c.left;
      if (++c.tau == c.s.n && c.left > 0) cursor_next_item(p, tab, c);
    }
    if (lane == 0 && *abort_flag) {
      // wait (bounded) for the copies this CTA issued before leaving
      for (uint32_t j = (it > STAGES ? it - STAGES : 0); j < it; ++j)
        mbar_wait_timed(&full[j % STAGES], (j / STAGES) & 1);
    }
    return;
  }

  // --------------------------------------------------------------------- compute warps
  // Per tile the warp computes S^T = K Q^T over its D slice (keys as M = 16, the CTA's query
  // rows as N in 8-row blocks), the slices are summed through shared memory, and
  // O^T += V^T P^T over the slice (D columns as M, rows as N, the tile's keys as K).  In the
  // accumulator layout a lane holds keys kr and kr + 8 (S^T) or D columns kr and kr + 8 (O^T),
  // each for query rows rq and rq + 1 of every 8-row block.
  const int dg = warp - C::MATH_WARP0;
  const int kr = lane >> 2;
  const int rq = 2 * (lane & 3);
  const int row0 = rg * C::ROWS;  // first query row of the item this CTA takes
  const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(p.q);

  Cursor c;
  cursor_begin(p, tab, start, end - start, c);
  uint32_t it = 0;
  int buf = 0;
  bool ok = true;
  while (c.left > 0 && ok) {
    // ---- segment setup: item (c.b, c.g), tiles [c.tau, seg_end)
    const int b = c.b, g = c.g;
    const int t_begin = c.tau;
    const long long rest = (long long)(c.s.n - c.tau);
    const int seg_n = (int)(c.left < rest ? c.left : rest);
    const bool whole = (t_begin == 0 && seg_n == c.s.n);
    const SeqRange s = c.s;

    // Q^T as the B operand: block nb holds query row row0 + nb*8 + kr, columns rq, rq + 1
    // (and + 8) of each 16-column step
    uint32_t qb[DS / 16][NB][2];
#pragma unroll
    for (int ks = 0; ks < DS / 16; ++ks)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = row0 + nb * 8 + kr;
          const int col = dg * DS + ks * 16 + rq + 8 * h;
          uint32_t v = 0;
          if (row < p.M) {
            const int j = row / p.G, hh = row % p.G;
            const size_t off =
                (((size_t)b * p.n_q + j) * p.Hq + (size_t)g * p.G + hh) * D + col;
            v = *reinterpret_cast<const uint32_t *>(qg + off);
          }
          qb[ks][nb][h] = v;
        }
    // keys every real row of this CTA may read: tiles inside [lo_all, hi_all] need no mask
    int lo_all = 1, hi_all = 0;
    {
      const int r_last = min(row0 + C::ROWS, p.M) - 1;
      if (r_last >= row0) {
        int lo_a, hi_a, lo_b, hi_b;
        row_range(p, s, b, row0, lo_a, hi_a);
        row_range(p, s, b, r_last, lo_b, hi_b);
        lo_all = max(lo_a, lo_b);
        hi_all = min(hi_a, hi_b);
      }
    }

    float m_run[NB][2], l_run[NB][2];
    float o[DS / 16][NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      m_run[nb][0] = m_run[nb][1] = -INFINITY;
      l_run[nb][0] = l_run[nb][1] = 0.f;
#pragma unroll
      for (int mb = 0; mb < DS / 16; ++mb)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[mb][nb][e] = 0.f;
    }

    // ---- partial S^T = K Q^T of one tile over this warp's D slice (with the registers of the
    // warpgroup split, even and odd 16-column steps in separate accumulators: two dependency
    // chains of half the length)
    constexpr int NCH = C::WS ? 2 : 1;
    auto qk_tile = [&](uint32_t kb, float (&part)[NB][4]) {
      float s2[NCH][NB][4];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
#pragma unroll
          for (int c = 0; c < NCH; ++c) s2[c][nb][e] = 0.f;
        }
      const int key = (lane & 7) + ((lane >> 3) & 1) * 8;
      const int coff = (lane >> 4) * 8;
#pragma unroll
      for (int ks = 0; ks < DS / 16; ++ks) {
        uint32_t ka[4];
        ldsm_x4(ka, kb + swz(key, dg * DS + ks * 16 + coff));
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
          mma_bf16_16816(s2[ks % NCH][nb], ka, qb[ks][nb][0], qb[ks][nb][1]);
      }
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          part[nb][e] = s2[0][nb][e];
#pragma unroll
          for (int c = 1; c < NCH; ++c) part[nb][e] += s2[c][nb][e];
        }
    };
    // (the warp leaves a wait together: its later shuffles and votes need every lane)
    auto wait_full = [&](uint32_t itx) {
      return __all_sync(0xffffffffu,
                        mbar_wait(&full[itx % STAGES], (itx / STAGES) & 1, abort_flag));
    };
    auto stage_k = [&](uint32_t itx) {
      return smem_u32(stages + (size_t)(itx % STAGES) * C::STAGE_BYTES);
    };
    // With several D slices and one row block (the drafter's call) the partials of tile t + 1
    // are computed and published before the exchange of tile t is awaited: the wait for the
    // other warps overlaps this warp's next products, nxt holding them in between (D 512,
    // B 8: 168.6 -> 163.5 us).  With more row blocks the extra live registers cost more than
    // the overlap gains (k 6: 270 -> 279 us), so those tiles keep the plain order.
    constexpr bool PIPE = NDG > 1 && NB == 1;
    static_assert(!PIPE || STAGES >= 2, "the next tile is awaited before this one is released");
    auto publish = [&](int bf, const float (&part)[NB][4]) {
      float4 *myred = reinterpret_cast<float4 *>(red) + ((bf * NCW + dg) * 32 + lane) * NB;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
        myred[nb] = make_float4(part[nb][0], part[nb][1], part[nb][2], part[nb][3]);
      mbar_arrive(&red_bar[bf]);
    };
    if constexpr (PIPE) {
      if (seg_n > 0) {
        if (!wait_full(it)) {
          record_status(p.status, SD_ERR_TIMEOUT);
          *abort_flag = 1;
          ok = false;
        } else {
          float part[NB][4];
          qk_tile(stage_k(it), part);
          publish(buf, part);
        }
      }
    }

    for (int t = 0; t < seg_n && ok; ++t) {
      const int stage = it % STAGES;
      if constexpr (!PIPE) {
        if (!wait_full(it)) {
          record_status(p.status, SD_ERR_TIMEOUT);
          *abort_flag = 1;
          ok = false;
          break;
        }
      }
      const int is_bad = bad[stage];
      const uint32_t kbase = smem_u32(stages + (size_t)stage * C::STAGE_BYTES);
      const uint32_t vbase = kbase + C::TILE_BYTES;
      const int p0 = (s.tf + t_begin + t) * kTile;

      float sc[NB][4];
      float nxt[PIPE ? NB : 1][4];
      const bool have_next = PIPE && t + 1 < seg_n;
      if constexpr (!PIPE) {
        qk_tile(kbase, sc);
        if constexpr (NDG > 1) publish(buf, sc);
      } else {
        if (have_next) {
          if (!wait_full(it + 1)) {
            record_status(p.status, SD_ERR_TIMEOUT);
            *abort_flag = 1;
            ok = false;
            break;
          }
          qk_tile(stage_k(it + 1), nxt);
        }
      }
      if constexpr (NDG > 1) {
        if (!__all_sync(0xffffffffu, mbar_wait(&red_bar[buf], (it >> 1) & 1, abort_flag))) {
          record_status(p.status, SD_ERR_TIMEOUT);
          *abort_flag = 1;
          ok = false;
          break;
        }
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[nb][e] = 0.f;
#pragma unroll
        for (int dd = 0; dd < NDG; ++dd) {
          const float4 *src = reinterpret_cast<const float4 *>(red) + ((buf * NCW + dd) * 32 + lane) * NB;
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const float4 a = src[nb];
            sc[nb][0] += a.x;
            sc[nb][1] += a.y;
            sc[nb][2] += a.z;
            sc[nb][3] += a.w;
          }
        }
        buf ^= 1;
      }

      // ---- scale (base-2 exponent), mask on the tiles that need it
      if (!is_bad && p0 >= lo_all && p0 + kTile - 1 <= hi_all) {
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[nb][e] *= p.scale_log2;
      } else {
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            int lo, hi;
            row_range(p, s, b, row0 + nb * 8 + rq + h, lo, hi);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              const int pos = p0 + kr + 8 * kk;
              const bool valid = !is_bad && pos >= lo && pos <= hi;
              sc[nb][2 * kk + h] = valid ? sc[nb][2 * kk + h] * p.scale_log2 : -INFINITY;
            }
          }
      }

      // ---- online softmax, rescaled lazily: a row's exponent base moves only when a tile's
      // maximum passes it by more than kRescale (the unscaled terms then stay below
      // 2^kRescale), so the accumulators are rescaled on few tiles
      {
        float xm[NB][2];
        bool grow = false;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            xm[nb][h] = fmaxf(sc[nb][h], sc[nb][h + 2]);
            grow |= xm[nb][h] > m_run[nb][h] + kRescale;
          }
        if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
          for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              float x = xm[nb][h];
              x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
              x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
              x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
              if (x > m_run[nb][h] + kRescale) {  // a finite maximum always passes -inf
                const float alpha =
                    m_run[nb][h] == -INFINITY ? 0.f : ex2_approx(m_run[nb][h] - x);
                m_run[nb][h] = x;
                l_run[nb][h] *= alpha;
#pragma unroll
                for (int mb = 0; mb < DS / 16; ++mb) {
                  o[mb][nb][h] *= alpha;
                  o[mb][nb][h + 2] *= alpha;
                }
              }
            }
        }
      }
      uint32_t pb[NB][2];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        float pv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float base = m_run[nb][e & 1] == -INFINITY ? 0.f : m_run[nb][e & 1];
          pv[e] = ex2_approx(sc[nb][e] - base);
          l_run[nb][e & 1] += pv[e];
        }
        // P^T (keys x rows, this lane: keys kr / kr + 8, rows rq, rq + 1) transposed in
        // registers into the B operand (keys rq, rq + 1 / + 8, row kr)
        pb[nb][0] = movmatrix_trans(pack_bf16x2(pv[0], pv[1]));
        pb[nb][1] = movmatrix_trans(pack_bf16x2(pv[2], pv[3]));
      }

      // ---- V rows no query of the item may read can hold anything (rolled-back or never
      // written slots, NaN included); zero this warp's slice of them so 0 * V stays 0.
      {
        int zlo = max(0, min(kTile, s.lo_min - p0));
        int zhi = max(0, min(kTile, s.hi_max - p0 + 1));
        if (is_bad) {
          zlo = kTile;
          zhi = kTile;
        }
        if (zlo > 0 || zhi < kTile) {
          uint8_t *vt = stages + (size_t)stage * C::STAGE_BYTES + C::TILE_BYTES;
          // rows [0, zlo) and [zhi, 16); slice columns [dg*DS, dg*DS+DS) = DS/64 chunks
          for (int u = lane; u < kTile * (DS / 64) * 8; u += 32) {
            const int row = u / ((DS / 64) * 8);
            const int rem = u % ((DS / 64) * 8);
            const int chunk = dg * (DS / 64) + rem / 8;
            const int unit = rem % 8;
            if (row < zlo || row >= zhi)
              *reinterpret_cast<uint4 *>(vt + chunk * (kTile * 128) + row * 128 + unit * 16) =
                  make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();  // before the stage is handed back to TMA
          __syncwarp();
        }
      }

      // ---- O^T += V^T P^T over this warp's D slice
      {
        const int key = (lane & 7) + (lane >> 4) * 8;
        const int coff = ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int mb = 0; mb < DS / 16; ++mb) {
          uint32_t va[4];
          ldsm_x4_trans(va, vbase + swz(key, dg * DS + mb * 16 + coff));
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) mma_bf16_16816(o[mb][nb], va, pb[nb][0], pb[nb][1]);
        }
      }
      mbar_arrive(&empty[stage]);
      if constexpr (PIPE) {
        if (have_next) publish(buf, nxt);  // buf was toggled after this tile's exchange
      }
      ++it;
    }
    if (!ok) break;

    // ---- segment end: final rows or a partial for the combine kernel
    float l_tot[NB][2];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float l = l_run[nb][h];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        l_tot[nb][h] = l;
      }
    if (whole) {
      __nv_bfloat16 *outg = reinterpret_cast<__nv_bfloat16 *>(p.out);
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = row0 + nb * 8 + rq + h;
          if (row >= p.M) continue;
          const int j = row / p.G, hh = row % p.G;
          const float inv = l_tot[nb][h] > 0.f ? 1.f / l_tot[nb][h] : 0.f;
          __nv_bfloat16 *dst =
              outg + (((size_t)b * p.n_q + j) * p.Hq + (size_t)g * p.G + hh) * D + dg * DS + kr;
#pragma unroll
          for (int mb = 0; mb < DS / 16; ++mb) {
            dst[mb * 16] = __float2bfloat16_rn(o[mb][nb][h] * inv);
            dst[mb * 16 + 8] = __float2bfloat16_rn(o[mb][nb][h + 2] * inv);
          }
        }
    } else {
      const size_t slot = (size_t)b * p.Hkv + g + grp;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = row0 + nb * 8 + rq + h;
          if (row >= p.M) continue;
          float *dst = p.ws_o + (slot * p.Mpad + row) * D + dg * DS + kr;
#pragma unroll
          for (int mb = 0; mb < DS / 16; ++mb) {
            dst[mb * 16] = o[mb][nb][h];
            dst[mb * 16 + 8] = o[mb][nb][h + 2];
          }
          if (dg == 0 && kr == 0) {
            p.ws_ml[(slot * p.Mpad + row) * 2 + 0] = m_run[nb][h];
            p.ws_ml[(slot * p.Mpad + row) * 2 + 1] = l_tot[nb][h];
          }
        }
    }
    c.tau += seg_n;
    c.left -= seg_n;
    if (c.left > 0) cursor_next_item(p, tab, c);
  }
}

// ------------------------------------------------------------ short key ranges (clusters)
// Sliding-window layers read at most window + n_q - 1 keys per item, too few to amortise a
// separate merge kernel.  A cluster of CS CTAs takes one item (sequence b, kv head g); CTA
// rank r streams tiles [n r / CS, n (r+1) / CS) of it, all of them in flight at once where the
// shared-memory ring holds them.  Inside a CTA, KG key groups of warps take the CTA's tiles
// round robin, each with its own online softmax.  Each CTA merges its KG partials (m, l, o) in
// key-group order and pushes the result, column slice by column slice, into the shared memory
// of the CTA owning that slice (CTA r owns output columns [D r / CS, D (r+1) / CS)); after one
// cluster barrier every CTA merges the CS partials of its slice in rank order and writes it.
// No workspace, one launch per call.

template <int D, int MT>
struct WCfg {
  static constexpr int DS = D >= 128 ? 128 : 64;
  static constexpr int NDG = D / DS;
  static constexpr int WPG = MT * NDG;                  // warps of one key group
  // key groups per CTA: at most 7 warps with two 16x128 slices or more per warp group, so the
  // register file of a sub-partition holds two warps of 255 registers (no spills)
  static constexpr int KG = WPG == 1 ? 8 : (6 / WPG > 0 ? 6 / WPG : 1);
  static constexpr int NCW = KG * WPG;
  static constexpr int THREADS = 32 * (NCW + 1);
  static constexpr int MP = 16 * MT;  // padded rows of an item
  static constexpr int MAX_CS = 8;    // CTAs per cluster at most
  static constexpr int TILE_BYTES = kTile * D * 2;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int RED_FLOATS = 2 * NCW * 32 * 8;
  static constexpr int ML_FLOATS = KG * MP * 2;       // key-group (m, l) partials
  static constexpr int RECV_FLOATS = MP * D;          // [CS][MP][D / CS] pushed column slices
  static constexpr int RECV_ML_FLOATS = MAX_CS * MP * 2;
  static constexpr size_t PART_BYTES = (size_t)KG * MP * D * 4;
  static constexpr size_t FIXED = 1024 + (size_t)(RED_FLOATS + ML_FLOATS + RECV_FLOATS +
                                                  RECV_ML_FLOATS) * 4 + 8 * (2 * 16 + 2 * KG + 1) +
                                  4 * (1 + 16) + 16;
  // A multiple of KG: tiles t and t + STAGES share a stage and belong to the same key group,
  // which consumes them in order (so a parity wait never sees the stage's previous phase).
  static constexpr int RING = (227 * 1024 - FIXED) / STAGE_BYTES > 16
                                  ? 16
                                  : (int)((227 * 1024 - FIXED) / STAGE_BYTES);
  static constexpr int STAGES = RING / KG * KG;
  static_assert(STAGES >= KG, "at least one stage per key group");
  static_assert(PART_BYTES <= (size_t)STAGES * STAGE_BYTES, "partials reuse the tile ring");
  static constexpr size_t SMEM = FIXED + (size_t)STAGES * STAGE_BYTES;
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

template <int D, int MT>
__global__ void __launch_bounds__(WCfg<D, MT>::THREADS, 1)
    attn_window_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap, const Params p, int CS) {
  using C = WCfg<D, MT>;
  constexpr int DS = C::DS, NDG = C::NDG, WPG = C::WPG, KG = C::KG, NCW = C::NCW;
  constexpr int STAGES = C::STAGES, MP = C::MP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *stages = smem;
  float *red = reinterpret_cast<float *>(smem + (size_t)STAGES * C::STAGE_BYTES);
  float *ml = red + C::RED_FLOATS;  // [KG][MP][2] partial (m, l) per row
  float *recv = ml + C::ML_FLOATS;  // [CS][MP][D / CS] partials of this CTA's column slice
  float *recv_ml = recv + C::RECV_FLOATS;  // [CS][MP][2]
  uint64_t *full = reinterpret_cast<uint64_t *>(recv_ml + C::RECV_ML_FLOATS);
  uint64_t *empty = full + STAGES;
  uint64_t *red_bar = empty + STAGES;  // [KG][2]
  uint64_t *done_bar = red_bar + 2 * KG;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(done_bar + 1);
  volatile int *bad = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int item = blockIdx.x / CS;
  const int b = item / p.Hkv, g = item % p.Hkv;
  pdl_trigger();
  pdl_wait();
  // one barrier per thread (full[], empty[], red_bar[], done_bar are contiguous), while the
  // loads of the sequence's range and the tensor-map prefetch are in flight
  {
    constexpr int NB = 2 * STAGES + 2 * KG + 1;
    const int i = threadIdx.x;
    if (i < NB) {
      const uint32_t cnt = i < STAGES ? 1u : (i < NB - 1 ? (uint32_t)(WPG * 32) : NCW * 32u);
      mbar_init(&full[i], cnt);
      fence_mbar_init();
    }
    if (i < STAGES) bad[i] = 0;
    if (i == 0) *abort_flag = 0;
  }
  if (warp == NCW && lane == 0) {
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
  }
  const SeqRange s = seq_range(p, b, threadIdx.x == 0 && g == 0 && rank == 0);
  __syncthreads();
  const int t_lo = (int)((long long)s.n * rank / CS);
  const int nl = (int)((long long)s.n * (rank + 1) / CS) - t_lo;

  if (warp == NCW) {
    // ------------------------------------------------------------------- producer warp
    // The whole warp walks the tiles; its lanes fetch the block-table entries of the next
    // 32 tiles at once, lane 0 issues the copies.
    int base = -32, blk_l = -1, t = 0;
    for (; t < nl; ++t) {
      if (t - base >= 32) {
        base = t;
        blk_l = -1;
        if (t + lane < nl) {
          const int bidx = (s.tf + t_lo + t + lane) * kTile / p.bs;
          if (bidx < p.mbps) blk_l = p.table[(size_t)b * p.mbps + bidx];
        }
      }
      const int blk = __shfl_sync(0xffffffffu, blk_l, t - base);
      int go = 1;
      if (lane == 0) {
        const int stage = t % STAGES;
        if (!mbar_wait(&empty[stage], ((t / STAGES) & 1) ^ 1, abort_flag)) {
          record_status(p.status, SD_ERR_TIMEOUT);
          *abort_flag = 1;
          go = 0;
        } else if (blk < 0 || blk >= p.num_blocks) {
          record_status(p.status, SD_ERR_DEVICE);
          bad[stage] = 1;
          mbar_arrive(&full[stage]);
        } else {
          bad[stage] = 0;
          const int p0 = (s.tf + t_lo + t) * kTile;
          const int row = (blk * p.Hkv + g) * p.bs + (p0 % p.bs);
          uint8_t *kd = stages + (size_t)stage * C::STAGE_BYTES;
          uint8_t *vd = kd + C::TILE_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          if (p.kv3d) {  // one box per tile brings every column chunk
            tma_load_3d(kd, &kmap, &full[stage], 0, row, 0);
            tma_load_3d(vd, &vmap, &full[stage], 0, row, 0);
          } else {
#pragma unroll
            for (int ch = 0; ch < D / 64; ++ch) {
              tma_load_2d(kd + ch * (kTile * 128), &kmap, &full[stage], ch * 64, row);
              tma_load_2d(vd + ch * (kTile * 128), &vmap, &full[stage], ch * 64, row);
            }
          }
        }
      }
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
    }
    if (lane == 0 && *abort_flag) {
      // wait (bounded) for the copies this CTA issued before its shared memory is reused
      for (int j = (t > STAGES ? t - STAGES : 0); j < t; ++j)
        mbar_wait_timed(&full[j % STAGES], (j / STAGES) & 1);
    }
    __syncwarp();
  } else {
    // --------------------------------------------------------------------- compute warps
    const int kg = warp / WPG, wi = warp % WPG, mg = wi / NDG, dg = wi % NDG;
    const int r0 = mg * 16 + (lane >> 2);
    const int kq = 2 * (lane & 3);
    const __nv_bfloat16 *qg = reinterpret_cast<const __nv_bfloat16 *>(p.q);
    uint32_t qa[DS / 16][4];
#pragma unroll
    for (int ks = 0; ks < DS / 16; ++ks) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = r0 + ((e & 1) ? 8 : 0);
        const int col = dg * DS + ks * 16 + kq + ((e & 2) ? 8 : 0);
        uint32_t v = 0;
        if (row < p.M && nl > 0) {
          const int j = row / p.G, hh = row % p.G;
          const size_t off = (((size_t)b * p.n_q + j) * p.Hq + (size_t)g * p.G + hh) * D + col;
          v = *reinterpret_cast<const uint32_t *>(qg + off);
        }
        qa[ks][e] = v;
      }
    }
    int lo0, hi0, lo1, hi1;
    row_range(p, s, b, r0, lo0, hi0);
    row_range(p, s, b, r0 + 8, lo1, hi1);

    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    float o[DS / 8][4];
#pragma unroll
    for (int nt = 0; nt < DS / 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;

    int j = 0;
    for (int t = kg; t < nl; t += KG, ++j) {
      const int stage = t % STAGES;
      // warp-uniform decisions: a lane that gave up must not leave the others in a shuffle
      if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], (t / STAGES) & 1, abort_flag))) {
        record_status(p.status, SD_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      const int buf = j & 1;
      const int is_bad = bad[stage];
      const uint32_t kbase = smem_u32(stages + (size_t)stage * C::STAGE_BYTES);
      const uint32_t vbase = kbase + C::TILE_BYTES;
      const int p0 = (s.tf + t_lo + t) * kTile;
      bool patched = false;
      if (MT == 1 && p.k_new != nullptr && !is_bad) {
        uint8_t *kt = stages + (size_t)stage * C::STAGE_BYTES;
        patched = patch_new_rows<D, DS>(p, b, g, s.L, p0, dg * DS, kt, kt + C::TILE_BYTES, lane);
      }

      // ---- partial S = Q K^T over this warp's D slice, summed over the key group's slices
      float sp[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sp[nt][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < DS / 16; ++ks) {
        const int d0 = dg * DS + ks * 16;
        uint32_t kb[4];
        const int key = ((lane >> 4) << 3) + (lane & 7);
        const int col = d0 + ((lane >> 3) & 1) * 8;
        ldsm_x4(kb, kbase + swz(key, col));
        mma_bf16_16816(sp[0], qa[ks], kb[0], kb[1]);
        mma_bf16_16816(sp[1], qa[ks], kb[2], kb[3]);
      }
      float sc[2][4];
      if (NDG == 1) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[nt][e] = sp[nt][e];
      } else {
        float *myred = red + ((size_t)((kg * 2 + buf) * WPG + wi) * 32 + lane) * 8;
        reinterpret_cast<float4 *>(myred)[0] =
            make_float4(sp[0][0], sp[0][1], sp[0][2], sp[0][3]);
        reinterpret_cast<float4 *>(myred)[1] =
            make_float4(sp[1][0], sp[1][1], sp[1][2], sp[1][3]);
        mbar_arrive(&red_bar[kg * 2 + buf]);
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&red_bar[kg * 2 + buf], (j >> 1) & 1, abort_flag))) {
          record_status(p.status, SD_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
#pragma unroll
        for (int dd = 0; dd < NDG; ++dd) {
          const float *src =
              red + ((size_t)((kg * 2 + buf) * WPG + mg * NDG + dd) * 32 + lane) * 8;
          const float4 a = reinterpret_cast<const float4 *>(src)[0];
          const float4 bq = reinterpret_cast<const float4 *>(src)[1];
          sc[0][0] += a.x;
          sc[0][1] += a.y;
          sc[0][2] += a.z;
          sc[0][3] += a.w;
          sc[1][0] += bq.x;
          sc[1][1] += bq.y;
          sc[1][2] += bq.z;
          sc[1][3] += bq.w;
        }
      }

      // ---- mask, online softmax (base-2 exponent with the scale folded in)
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int pos = p0 + nt * 8 + kq + (e & 1);
          const int lo = (e & 2) ? lo1 : lo0, hi = (e & 2) ? hi1 : hi0;
          const bool valid = !is_bad && pos >= lo && pos <= hi;
          const float x = valid ? sc[nt][e] * p.scale_log2 : -INFINITY;
          sc[nt][e] = x;
          mx[e >> 1] = fmaxf(mx[e >> 1], x);
        }
      if constexpr (MT == 1) {
        // one query tile: the kernel streams at the memory's pace, rescale every tile
        float alpha[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
          mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
          const float m_new = fmaxf(m_run[h], mx[h]);
          const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
          alpha[h] = exp2f(m_run[h] - m_use);
          m_run[h] = m_new;
          l_run[h] *= alpha[h];
          mx[h] = m_use;
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float pv = exp2f(sc[nt][e] - mx[e >> 1]);
            sc[nt][e] = pv;
            l_run[e >> 1] += pv;
          }
#pragma unroll
        for (int nt = 0; nt < DS / 8; ++nt) {
          o[nt][0] *= alpha[0];
          o[nt][1] *= alpha[0];
          o[nt][2] *= alpha[1];
          o[nt][3] *= alpha[1];
        }
      } else {
        // several query tiles make the kernel issue-bound: a row's exponent base moves only
        // when a tile's maximum passes it by more than kRescale (the unscaled terms then stay
        // below 2^kRescale), so the accumulators are rescaled on few tiles and the warp skips
        // the rescale otherwise
        bool grow = false;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
          mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
          grow |= mx[h] > m_run[h] + kRescale;
        }
        if (__any_sync(0xffffffffu, grow)) {
          float alpha[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            alpha[h] = 1.f;
            if (mx[h] > m_run[h] + kRescale) {  // a finite maximum always passes -inf
              alpha[h] = m_run[h] == -INFINITY ? 0.f : ex2_approx(m_run[h] - mx[h]);
              m_run[h] = mx[h];
            }
            l_run[h] *= alpha[h];
          }
#pragma unroll
          for (int nt = 0; nt < DS / 8; ++nt) {
            o[nt][0] *= alpha[0];
            o[nt][1] *= alpha[0];
            o[nt][2] *= alpha[1];
            o[nt][3] *= alpha[1];
          }
        }
        const float base0 = m_run[0] == -INFINITY ? 0.f : m_run[0];
        const float base1 = m_run[1] == -INFINITY ? 0.f : m_run[1];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float pv = ex2_approx(sc[nt][e] - ((e & 2) ? base1 : base0));
            sc[nt][e] = pv;
            l_run[e >> 1] += pv;
          }
      }
      uint32_t pa[4];
      pa[0] = pack_bf16x2(sc[0][0], sc[0][1]);
      pa[1] = pack_bf16x2(sc[0][2], sc[0][3]);
      pa[2] = pack_bf16x2(sc[1][0], sc[1][1]);
      pa[3] = pack_bf16x2(sc[1][2], sc[1][3]);

      // ---- V rows no query of the item may read can hold anything (rolled-back or never
      // written slots, NaN included); zero this warp's slice of them so 0 * V stays 0.
      {
        int zlo = max(0, min(kTile, s.lo_min - p0));
        int zhi = max(0, min(kTile, s.hi_max - p0 + 1));
        if (is_bad) {
          zlo = kTile;
          zhi = kTile;
        }
        if (zlo > 0 || zhi < kTile) {
          uint8_t *vt = stages + (size_t)stage * C::STAGE_BYTES + C::TILE_BYTES;
          for (int u = lane; u < kTile * (DS / 64) * 8; u += 32) {
            const int row = u / ((DS / 64) * 8);
            const int rem = u % ((DS / 64) * 8);
            const int chunk = dg * (DS / 64) + rem / 8;
            const int unit = rem % 8;
            if (row < zlo || row >= zhi)
              *reinterpret_cast<uint4 *>(vt + chunk * (kTile * 128) + row * 128 + unit * 16) =
                  make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
          patched = false;
        }
        if (patched) fence_proxy_async_smem();
      }

      // ---- O += P V over this warp's D slice
#pragma unroll
      for (int np = 0; np < DS / 16; ++np) {
        const int d0 = dg * DS + np * 16;
        uint32_t vb[4];
        const int key = ((lane >> 3) & 1) * 8 + (lane & 7);
        const int col = d0 + (lane >> 4) * 8;
        ldsm_x4_trans(vb, vbase + swz(key, col));
        mma_bf16_16816(o[2 * np], pa, vb[0], vb[1]);
        mma_bf16_16816(o[2 * np + 1], pa, vb[2], vb[3]);
      }
      mbar_arrive(&empty[stage]);
    }
    float l_tot[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float l = l_run[h];
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      l_tot[h] = l;
    }
    // every compute warp is done with the tile ring before it holds the partials
    mbar_arrive(done_bar);
    if (!mbar_wait(done_bar, 0, abort_flag)) {
      record_status(p.status, SD_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    float *po = reinterpret_cast<float *>(stages);  // [KG][MP][D]
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = r0 + 8 * h;
      if (row >= p.M) continue;
      float *dst = po + ((size_t)kg * MP + row) * D + dg * DS + kq;
#pragma unroll
      for (int nt = 0; nt < DS / 8; ++nt)
        *reinterpret_cast<float2 *>(dst + nt * 8) = make_float2(o[nt][2 * h], o[nt][2 * h + 1]);
      if (dg == 0 && (lane & 3) == 0)
        *reinterpret_cast<float2 *>(ml + ((size_t)kg * MP + row) * 2) =
            make_float2(m_run[h], l_tot[h]);
    }
  }
  __syncthreads();

  // ---- key-group merge of each (row, 4 columns), pushed to the CTA owning the columns
  const int cols = D / CS;
  for (int u = threadIdx.x; u < p.M * (D / 4); u += C::THREADS) {
    const int row = u / (D / 4), col = (u % (D / 4)) * 4;
    float2 mlv[KG];
    float4 ov[KG];
#pragma unroll
    for (int k = 0; k < KG; ++k) {
      mlv[k] = *reinterpret_cast<const float2 *>(ml + ((size_t)k * MP + row) * 2);
      ov[k] = *reinterpret_cast<const float4 *>(
          reinterpret_cast<const float *>(stages) + ((size_t)k * MP + row) * D + col);
    }
    float m_acc = -INFINITY, l_acc = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < KG; ++k) {
      if (mlv[k].x == -INFINITY) continue;
      const float m_new = fmaxf(m_acc, mlv[k].x);
      const float a = exp2f(m_acc - m_new), w = exp2f(mlv[k].x - m_new);
      l_acc = l_acc * a + mlv[k].y * w;
      acc.x = acc.x * a + ov[k].x * w;
      acc.y = acc.y * a + ov[k].y * w;
      acc.z = acc.z * a + ov[k].z * w;
      acc.w = acc.w * a + ov[k].w * w;
      m_acc = m_new;
    }
    const int owner = col / cols, cc = col % cols;
    st_dsmem_f4(dsmem_addr(smem_u32(recv + ((size_t)rank * MP + row) * cols + cc), owner), acc);
    if (cc == 0)
      st_dsmem_f2(dsmem_addr(smem_u32(recv_ml + ((size_t)rank * MP + row) * 2), owner),
                  make_float2(m_acc, l_acc));
  }
  cluster_sync();  // every CTA's pushes have landed; nothing below touches another CTA

  // ---- this CTA's column slice: the CS partials merged in rank order
  __nv_bfloat16 *outg = reinterpret_cast<__nv_bfloat16 *>(p.out);
  for (int u = threadIdx.x; u < p.M * (cols / 4); u += C::THREADS) {
    const int row = u / (cols / 4), cc = (u % (cols / 4)) * 4;
    float m_acc = -INFINITY, l_acc = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < CS; ++q) {
      const float2 mlq = *reinterpret_cast<const float2 *>(recv_ml + ((size_t)q * MP + row) * 2);
      if (mlq.x == -INFINITY) continue;
      const float4 oq =
          *reinterpret_cast<const float4 *>(recv + ((size_t)q * MP + row) * cols + cc);
      const float m_new = fmaxf(m_acc, mlq.x);
      const float a = exp2f(m_acc - m_new), w = exp2f(mlq.x - m_new);
      l_acc = l_acc * a + mlq.y * w;
      acc.x = acc.x * a + oq.x * w;
      acc.y = acc.y * a + oq.y * w;
      acc.z = acc.z * a + oq.z * w;
      acc.w = acc.w * a + oq.w * w;
      m_acc = m_new;
    }
    const float inv = l_acc > 0.f ? 1.f / l_acc : 0.f;
    const int jq = row / p.G, hh = row % p.G;
    __nv_bfloat16 *dst = outg + (((size_t)b * p.n_q + jq) * p.Hq + (size_t)g * p.G + hh) * D +
                         (int)rank * cols + cc;
    *reinterpret_cast<uint2 *>(dst) =
        make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
  }
}

// Merges the partials of items that several CTAs shared; writes zero rows for drafter items
// with an empty key range.  One CTA per (item, query row) of G groups of 128 threads (4
// columns a thread): the groups take runs of 8 partials in turn, and the group sums are added
// in group order (a fixed order for a given partition of the tiles and G).  More groups
// shorten the chain of dependent loads when an item has many partials; the host picks them
// when the CTAs still fit one wave.
template <typename T, int G>
__global__ void __launch_bounds__(128 * G) attn_combine_kernel(const Params p) {
  constexpr int kChunk = 512;
  __shared__ long long s_F, s_Fl, s_T;
  __shared__ int s_n;
  __shared__ float s_w[kChunk];
  __shared__ float s_red[4 * G];
  __shared__ float4 s_acc[G > 1 ? G - 1 : 1][128];
  pdl_trigger();
  pdl_wait();
  const int item = blockIdx.x, row = blockIdx.y;
  const int b = item / p.Hkv, g = item % p.Hkv;
  if (threadIdx.x < 32) {  // tile counts of all sequences, one warp
    long long pre = 0, T_all = 0;
    int n = 0;
    for (int bb = threadIdx.x; bb < p.B; bb += 32) {
      SeqRange sr = seq_range(p, bb, bb == b && g == 0 && row == 0);
      if (bb == b) n = sr.n;
      if (bb < b) pre += (long long)p.Hkv * sr.n;
      T_all += (long long)p.Hkv * sr.n;
    }
    for (int o = 16; o > 0; o >>= 1) {
      pre += __shfl_xor_sync(0xffffffffu, pre, o);
      T_all += __shfl_xor_sync(0xffffffffu, T_all, o);
      n += __shfl_xor_sync(0xffffffffu, n, o);
    }
    if (threadIdx.x == 0) {
      s_n = n;
      s_F = pre + (long long)g * n;
      s_Fl = s_F + n - 1;
      s_T = T_all;
    }
  }
  __syncthreads();
  const int j = row / p.G, hh = row % p.G;
  T *dst = reinterpret_cast<T *>(p.out) +
           (((size_t)b * p.n_q + j) * p.Hq + (size_t)g * p.G + hh) * p.D;
  if (s_n == 0) {
    for (int d = threadIdx.x; d < p.D; d += blockDim.x) dst[d] = T(0.f);
    return;
  }
  const long long F = s_F, Fl = s_Fl, T_all = s_T;
  const int c_first = (int)(((F + 1) * p.P - 1) / T_all);
  const int c_last = (int)(((Fl + 1) * p.P - 1) / T_all);
  if (c_first == c_last) return;  // written directly by its only CTA
  const size_t slot0 = (size_t)b * p.Hkv + g;
  // CTA c holds tiles [T*c/P, T*(c+1)/P); with fewer tiles than CTAs some hold none and
  // wrote no partial for this item.
  auto holds = [&](int c) {
    const long long s_c = T_all * c / p.P, e_c = T_all * (c + 1) / p.P;
    return e_c > F && s_c <= Fl && e_c > s_c;
  };
  auto block_reduce = [&](float v, bool is_max) {
    for (int o = 16; o > 0; o >>= 1) {
      const float u = __shfl_xor_sync(0xffffffffu, v, o);
      v = is_max ? fmaxf(v, u) : v + u;
    }
    __syncthreads();
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = s_red[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = is_max ? fmaxf(r, s_red[w]) : r + s_red[w];
    return r;
  };
  const int S = c_last - c_first + 1;
  float mloc = -INFINITY;
  for (int t = threadIdx.x; t < S; t += blockDim.x)
    if (holds(c_first + t))
      mloc = fmaxf(mloc, p.ws_ml[((slot0 + c_first + t) * p.Mpad + row) * 2]);
  const float mmax = block_reduce(mloc, true);
  float den_loc = 0.f;
  if (mmax != -INFINITY)
    for (int t = threadIdx.x; t < S; t += blockDim.x)
      if (holds(c_first + t)) {
        const size_t sl = (slot0 + c_first + t) * p.Mpad + row;
        den_loc += exp2f(p.ws_ml[sl * 2] - mmax) * p.ws_ml[sl * 2 + 1];
      }
  const float den = block_reduce(den_loc, false);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  // weighted sum of the partial rows, kChunk slots at a time; group grp takes runs of 8
  // slots u0 = 8 grp, 8 (grp + G), ..., the loads of a run issued before its multiply-adds
  // (they are independent L2 reads)
  const int grp = threadIdx.x >> 7, tid = threadIdx.x & 127;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};  // D <= 512: 4 columns per thread of a group
  for (int t0 = 0; t0 < S; t0 += kChunk) {
    const int n = min(kChunk, S - t0);
    __syncthreads();
    for (int t = threadIdx.x; t < n; t += blockDim.x) {
      const int c = c_first + t0 + t;
      s_w[t] = (mmax != -INFINITY && holds(c))
                   ? exp2f(p.ws_ml[((slot0 + c) * p.Mpad + row) * 2] - mmax)
                   : 0.f;
    }
    __syncthreads();
    for (int u0 = 8 * grp; u0 < n; u0 += 8 * G) {
      float v[8][4];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float w = u0 + u < n ? s_w[u0 + u] : 0.f;
        const float *o = p.ws_o + ((slot0 + c_first + t0 + u0 + u) * p.Mpad + row) * p.D;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int d = tid + e * 128;
          v[u][e] = (w != 0.f && d < p.D) ? __ldcg(o + d) : 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float w = u0 + u < n ? s_w[u0 + u] : 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] = fmaf(w, v[u][e], acc[e]);
      }
    }
  }
  if constexpr (G > 1) {
    if (grp > 0) s_acc[grp - 1][tid] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    __syncthreads();
    if (grp > 0) return;
#pragma unroll
    for (int g2 = 0; g2 < G - 1; ++g2) {
      const float4 a = s_acc[g2][tid];
      acc[0] += a.x;
      acc[1] += a.y;
      acc[2] += a.z;
      acc[3] += a.w;
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int d = tid + e * 128;
    if (d < p.D) dst[d] = T(acc[e] * inv);
  }
}

// Writes the n_q new K/V rows of every sequence into the cache (verify only).  The h_kv rows
// of one position are h_kv * D contiguous elements both in k_new and in the cache block.
template <typename T>
__global__ void append_kv_kernel(const Params p, const T *k_new, const T *v_new, T *k_cache,
                                 T *v_cache) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x / p.n_q, j = blockIdx.x % p.n_q;
  const int L = p.ctx_len[b];
  if (L < 0) return;  // reported by the attention kernel
  const int pos = L + j;
  const int bidx = pos / p.bs;
  if (bidx >= p.mbps) {
    if (threadIdx.x == 0) record_status(p.status, SD_ERR_DEVICE);
    return;
  }
  const int blk = p.table[(size_t)b * p.mbps + bidx];
  if (blk < 0 || blk >= p.num_blocks) {
    if (threadIdx.x == 0) record_status(p.status, SD_ERR_DEVICE);
    return;
  }
  constexpr int E = 16 / sizeof(T);  // elements per 16-byte vector (D is a multiple of E)
  const int per_head = p.D / E;
  const int n = p.Hkv * per_head;
  for (int idx = threadIdx.x; idx < n; idx += blockDim.x) {
    const int g = idx / per_head, e = idx % per_head;
    const size_t src = (((size_t)b * p.n_q + j) * p.Hkv + g) * per_head + e;
    const size_t dst = (((size_t)blk * p.Hkv + g) * p.bs + pos % p.bs) * per_head + e;
    reinterpret_cast<uint4 *>(k_cache)[dst] = reinterpret_cast<const uint4 *>(k_new)[src];
    reinterpret_cast<uint4 *>(v_cache)[dst] = reinterpret_cast<const uint4 *>(v_new)[src];
  }
}

// float32 path: one warp per (sequence, query position, head).
// One CTA per query row; warp w takes the row's keys lo + w, lo + w + kF32Warps, ... with the
// lanes over the head dimension.  The block ids of the next 32 keys of a warp are fetched
// lane-parallel, and the K and V rows of kF32Unroll keys are loaded together, so a warp has
// several keys' loads in flight.  Each warp keeps its own online softmax; the warps' (m, l, o)
// are merged in warp order through shared memory.
constexpr int kF32Warps = 8;
constexpr int kF32Unroll = 4;

__global__ void __launch_bounds__(32 * kF32Warps) attn_f32_kernel(const Params p,
                                                                  const float *k_cache,
                                                                  const float *v_cache) {
  __shared__ float s_ml[kF32Warps][2];
  __shared__ float s_o[kF32Warps][512];
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_id = blockIdx.x;  // (b, j, h)
  const int h = row_id % p.Hq;
  const int j = (row_id / p.Hq) % p.n_q;
  const int b = row_id / (p.Hq * p.n_q);
  const int g = h / p.G;
  const SeqRange s = seq_range(p, b, threadIdx.x == 0);
  int lo, hi;
  row_range(p, s, b, j * p.G + (h % p.G), lo, hi);
  constexpr int MAXE = 16;  // D <= 512
  const int per = p.D / 32;
  const float *qv =
      reinterpret_cast<const float *>(p.q) + (((size_t)b * p.n_q + j) * p.Hq + h) * p.D;
  float qr[MAXE], acc[MAXE];
#pragma unroll
  for (int e = 0; e < MAXE; ++e) {
    qr[e] = e < per ? qv[lane + 32 * e] : 0.f;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int nk = hi >= lo ? hi - lo + 1 : 0;
  const int mine = nk > warp ? (nk - warp + kF32Warps - 1) / kF32Warps : 0;  // this warp's keys
  for (int base = 0; base < mine; base += 32) {
    // block ids of keys base .. base + 31 of this warp, one per lane
    int blk_l = -1;
    if (base + lane < mine) {
      const int pos = lo + warp + kF32Warps * (base + lane);
      blk_l = p.table[(size_t)b * p.mbps + pos / p.bs];
      if (blk_l < 0 || blk_l >= p.num_blocks) {
        record_status(p.status, SD_ERR_DEVICE);
        blk_l = -1;
      }
    }
    const int cnt = min(32, mine - base);
    for (int i0 = 0; i0 < cnt; i0 += kF32Unroll) {
      float kr[kF32Unroll][MAXE], vr[kF32Unroll][MAXE];
      bool valid[kF32Unroll];
#pragma unroll
      for (int u = 0; u < kF32Unroll; ++u) {
        const int i = i0 + u;
        const int blk = __shfl_sync(0xffffffffu, blk_l, i < cnt ? i : 0);
        valid[u] = i < cnt && blk >= 0;
        const int pos = lo + warp + kF32Warps * (base + i);
        const size_t row = valid[u] ? (((size_t)blk * p.Hkv + g) * p.bs + pos % p.bs) * p.D : 0;
#pragma unroll
        for (int e = 0; e < MAXE; ++e) {
          kr[u][e] = (valid[u] && e < per) ? k_cache[row + lane + 32 * e] : 0.f;
          vr[u][e] = (valid[u] && e < per) ? v_cache[row + lane + 32 * e] : 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < kF32Unroll; ++u) {
        if (!valid[u]) continue;  // warp-uniform
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < MAXE; ++e) dot = fmaf(qr[e], kr[u][e], dot);
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        const float x = dot * p.scale;
        const float m_new = fmaxf(m, x);
        const float alpha = expf(m - m_new);
        const float w = expf(x - m_new);
        l = l * alpha + w;
#pragma unroll
        for (int e = 0; e < MAXE; ++e) acc[e] = acc[e] * alpha + w * vr[u][e];
        m = m_new;
      }
    }
  }
  // merge the warps in order
  if (lane == 0) {
    s_ml[warp][0] = m;
    s_ml[warp][1] = l;
  }
#pragma unroll
  for (int e = 0; e < MAXE; ++e)
    if (e < per) s_o[warp][lane + 32 * e] = acc[e];
  __syncthreads();
  if (warp != 0) return;
  float M = -INFINITY;
  for (int w = 0; w < kF32Warps; ++w) M = fmaxf(M, s_ml[w][0]);
  float L = 0.f, o[MAXE];
#pragma unroll
  for (int e = 0; e < MAXE; ++e) o[e] = 0.f;
  for (int w = 0; w < kF32Warps; ++w) {
    const float sc = s_ml[w][0] == -INFINITY ? 0.f : expf(s_ml[w][0] - M);
    L += s_ml[w][1] * sc;
#pragma unroll
    for (int e = 0; e < MAXE; ++e)
      if (e < per) o[e] += s_o[w][lane + 32 * e] * sc;
  }
  float *ov = reinterpret_cast<float *>(p.out) + (((size_t)b * p.n_q + j) * p.Hq + h) * p.D;
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int e = 0; e < MAXE; ++e)
    if (e < per) ov[lane + 32 * e] = o[e] * inv;
}

// ------------------------------------------------------------------------------- host side

template <int D, int NB, int STAGES, bool SPLIT>
struct Launcher {
  using C = Cfg<D, NB, STAGES, SPLIT>;
  static int ctas_per_sm() {
    static int dev_cache[64];
    static int occ_cache[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && dev_cache[dev] == dev + 1) return occ_cache[dev];
    cudaFuncSetAttribute(attn_bf16_kernel<D, NB, STAGES, SPLIT>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    cudaFuncSetAttribute(attn_bf16_kernel<D, NB, STAGES, SPLIT>,
                         cudaFuncAttributePreferredSharedMemoryCarveout,
                         (int)cudaSharedmemCarveoutMaxShared);
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, attn_bf16_kernel<D, NB, STAGES, SPLIT>,
                                                      C::THREADS, C::SMEM) != cudaSuccess)
      occ = 0;
    if constexpr (C::WS) {
      // the warpgroups' register split must match the registers the kernel launches with
      cudaFuncAttributes fa{};
      if (cudaFuncGetAttributes(&fa, attn_bf16_kernel<D, NB, STAGES, SPLIT>) != cudaSuccess ||
          fa.numRegs != C::kRegLaunch)
        occ = 0;
    }
    if (dev < 64) {
      occ_cache[dev] = occ;
      dev_cache[dev] = dev + 1;
    }
    return occ;
  }
  static sd_status launch(const CUtensorMap &km, const CUtensorMap &vm, const Params &p,
                          cudaStream_t st) {
    return cuda_status(
        sdv::launch(attn_bf16_kernel<D, NB, STAGES, SPLIT>, dim3(p.P * p.row_groups), dim3(C::THREADS),
                    C::SMEM, st,
                    km, vm, p));
  }
};

#define SDV_STAGES(D) ((D) == 512 ? 3 : (D) == 256 ? 4 : (D) == 128 ? 6 : 8)

// Persistent CTAs for a (head_dim, 8-row blocks, register split) case on the current device.
static int persistent_ctas(int D, const RowSplit &rs) {
  int occ = 0;
#define SDV_CASE(DD, NN, SS) \
  if (D == DD && rs.NB == NN && rs.split == SS) \
    occ = Launcher<DD, NN, SDV_STAGES(DD), SS>::ctas_per_sm();
  SDV_CASE(64, 1, false) SDV_CASE(128, 1, false) SDV_CASE(256, 1, false) SDV_CASE(512, 1, false)
  SDV_CASE(64, 2, false) SDV_CASE(128, 2, false) SDV_CASE(256, 2, false) SDV_CASE(512, 2, false)
  SDV_CASE(64, 3, false) SDV_CASE(128, 3, false) SDV_CASE(256, 3, false) SDV_CASE(512, 3, false)
  SDV_CASE(512, 2, true) SDV_CASE(512, 3, true)
#undef SDV_CASE
  const int sms = sm_count();
  if (occ <= 0 || sms <= 0) return 0;
  return occ * sms;
}

// Four combine groups when an item spreads over 32 or more CTAs (P CTA groups over `items`
// items of similar length) and one CTA per SM covers the grid of `ctas`; else one (with a few
// partials per item the extra groups only add scheduling: B 8, k 2, about 10 partials: 180 ->
// 182 us with two groups).
static bool combine_wide(int ctas, int P, int items) {
  const int sms = std::max(sm_count(), 1);
  return ctas <= sms && P >= 32 * items;
}

static sd_status launch_bf16(int D, const RowSplit &rs, const CUtensorMap &km,
                             const CUtensorMap &vm, const Params &p, cudaStream_t st) {
#define SDV_CASE(DD, NN, SS)                            \
  if (D == DD && rs.NB == NN && rs.split == SS)         \
    return Launcher<DD, NN, SDV_STAGES(DD), SS>::launch(km, vm, p, st);
  SDV_CASE(64, 1, false) SDV_CASE(128, 1, false) SDV_CASE(256, 1, false) SDV_CASE(512, 1, false)
  SDV_CASE(64, 2, false) SDV_CASE(128, 2, false) SDV_CASE(256, 2, false) SDV_CASE(512, 2, false)
  SDV_CASE(64, 3, false) SDV_CASE(128, 3, false) SDV_CASE(256, 3, false) SDV_CASE(512, 3, false)
  SDV_CASE(512, 2, true) SDV_CASE(512, 3, true)
#undef SDV_CASE
  return SD_ERR_UNSUPPORTED;
}

// Sliding windows up to this many keys take the cluster path (one launch, no workspace).
constexpr int kWinMax = 2048;

template <int D, int MT>
struct WLauncher {
  using C = WCfg<D, MT>;
  // Clusters of 1, 2, 4 and 8 CTAs resident at once on the current device.
  static const int *max_clusters() {
    static int cache[64][4];
    static int dev_ok[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && dev_ok[dev] == dev + 1) return cache[dev];
    static int scratch[4];
    int *out = dev < 64 ? cache[dev] : scratch;
    cudaFuncSetAttribute(attn_window_kernel<D, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)C::SMEM);
    for (int i = 0; i < 4; ++i) {
      const int cs = 1 << i;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(cs);
      cfg.blockDim = dim3(C::THREADS);
      cfg.dynamicSmemBytes = C::SMEM;
      cudaLaunchAttribute a[1];
      a[0].id = cudaLaunchAttributeClusterDimension;
      a[0].val.clusterDim.x = cs;
      a[0].val.clusterDim.y = 1;
      a[0].val.clusterDim.z = 1;
      cfg.attrs = a;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, attn_window_kernel<D, MT>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
      }
      out[i] = n;
    }
    if (dev < 64) dev_ok[dev] = dev + 1;
    return out;
  }
  static sd_status launch(const CUtensorMap &km, const CUtensorMap &vm, const Params &p,
                          int tiles_max, cudaStream_t st) {
    const int *mc = max_clusters();
    if (mc[0] <= 0) return SD_ERR_CUDA;
    const int items = p.B * p.Hkv;
    int cs = 1;
    for (int i = 3; i >= 1; --i)
      if ((1 << i) <= tiles_max && items <= mc[i]) {
        cs = 1 << i;
        break;
      }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(items * cs);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute a[2];
    a[0].id = cudaLaunchAttributeClusterDimension;
    a[0].val.clusterDim.x = cs;
    a[0].val.clusterDim.y = 1;
    a[0].val.clusterDim.z = 1;
    a[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = a;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, attn_window_kernel<D, MT>, km, vm, p, cs));
  }
};

static sd_status launch_window(int D, int MT, const CUtensorMap &km, const CUtensorMap &vm,
                               const Params &p, int tiles_max, cudaStream_t st) {
#define SDV_CASE(DD, MM) \
  if (D == DD && MT == MM) return WLauncher<DD, MM>::launch(km, vm, p, tiles_max, st);
  SDV_CASE(64, 1) SDV_CASE(64, 2) SDV_CASE(128, 1) SDV_CASE(128, 2)
  SDV_CASE(256, 1) SDV_CASE(256, 2) SDV_CASE(512, 1) SDV_CASE(512, 2)
#undef SDV_CASE
  return SD_ERR_UNSUPPORTED;
}

static sd_status validate(const sd_attn_desc *d, bool draft) {
  if (!d) return SD_ERR_INVALID_ARG;
  if (d->batch < 1 || d->n_q < 1 || d->h_q < 1 || d->h_kv < 1 || d->h_q % d->h_kv)
    return SD_ERR_INVALID_ARG;
  if (draft && d->n_q != 1) return SD_ERR_INVALID_ARG;
  if (d->block_size < 1 || d->max_blocks_per_seq < 1 || d->num_blocks < 1)
    return SD_ERR_INVALID_ARG;
  if (!(d->scale > 0.f) || d->scale != d->scale) return SD_ERR_INVALID_ARG;
  if ((long long)d->num_blocks * d->h_kv * d->block_size >= (1ll << 31))
    return SD_ERR_UNSUPPORTED;
  const int G = d->h_q / d->h_kv;
  if ((long long)G * d->n_q > 64) return SD_ERR_UNSUPPORTED;
  if (d->dtype == SD_BF16) {
    if (!(d->head_dim == 64 || d->head_dim == 128 || d->head_dim == 256 || d->head_dim == 512))
      return SD_ERR_UNSUPPORTED;
    if (d->block_size % 16) return SD_ERR_UNSUPPORTED;
  } else if (d->dtype == SD_F32) {
    if (d->head_dim < 32 || d->head_dim > 512 || d->head_dim % 32) return SD_ERR_UNSUPPORTED;
  } else {
    return SD_ERR_INVALID_ARG;
  }
  return SD_OK;
}

// Stream-K groups of the split-KV kernel: its persistent CTAs, divided into groups of one CTA
// per row group of the item.
static int grid_ctas(const sd_attn_desc *d) {
  if (d->dtype != SD_BF16) return 0;
  const RowSplit rs = row_split(d->h_q / d->h_kv * d->n_q, d->head_dim);
  return std::min(kMaxGroups, persistent_ctas(d->head_dim, rs) / rs.R);
}

static size_t ws_size(const sd_attn_desc *d) {
  if (validate(d, false) != SD_OK && validate(d, true) != SD_OK) return 0;
  if (d->dtype != SD_BF16) return 0;
  const RowSplit rs = row_split(d->h_q / d->h_kv * d->n_q, d->head_dim);
  const int Mpad = rs.R * 8 * rs.NB;
  const size_t slots = (size_t)d->batch * d->h_kv + (size_t)grid_ctas(d);
  return round_up(slots * Mpad * d->head_dim * 4, 256) + round_up(slots * Mpad * 2 * 4, 256);
}

static sd_status run(const sd_attn_desc *d, bool draft, const void *q, const void *k_new,
                     const void *v_new, void *k_cache, void *v_cache, const int32_t *table,
                     const int32_t *ctx_len, const int32_t *q_pos, void *out, void *ws,
                     size_t ws_bytes, cudaStream_t st) {
  sd_status s = validate(d, draft);
  if (s != SD_OK) return s;
  if (!q || !k_cache || !v_cache || !table || !ctx_len || !out) return SD_ERR_INVALID_ARG;
  if (!draft && (!k_new || !v_new)) return SD_ERR_INVALID_ARG;
  Params p{};
  p.B = d->batch;
  p.n_q = d->n_q;
  p.Hq = d->h_q;
  p.Hkv = d->h_kv;
  p.G = d->h_q / d->h_kv;
  p.D = d->head_dim;
  p.bs = d->block_size;
  p.mbps = d->max_blocks_per_seq;
  p.num_blocks = d->num_blocks;
  p.window = d->window > 0 ? d->window : 0;
  p.M = p.G * p.n_q;
  p.is_draft = draft ? 1 : 0;
  p.q_offset = d->q_offset;
  p.scale = d->scale;
  p.scale_log2 = d->scale * 1.4426950408889634f;
  p.q = q;
  p.table = table;
  p.ctx_len = ctx_len;
  p.q_pos = q_pos;
  p.out = out;
  p.status = device_status_word();

  if (d->dtype == SD_F32) {
    if (!draft) {
      if (launch(append_kv_kernel<float>, dim3(p.B * p.n_q), dim3(256), 0, st, p,
                 (const float *)k_new, (const float *)v_new, (float *)k_cache,
                 (float *)v_cache) != cudaSuccess)
        return SD_ERR_CUDA;
    }
    return cuda_status(launch(attn_f32_kernel, dim3(p.B * p.n_q * p.Hq), dim3(32 * kF32Warps),
                              0, st, p, (const float *)k_cache, (const float *)v_cache));
  }

  // bf16
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      (!draft && (!aligned16(k_new) || !aligned16(v_new))))
    return SD_ERR_INVALID_ARG;
  const int MT = (p.M + 15) / 16;  // 16-row query tiles of the cluster (sliding-window) kernel
  const RowSplit rs = row_split(p.M, p.D);
  p.row_groups = rs.R;
  p.Mpad = rs.R * 8 * rs.NB;
  p.P = grid_ctas(d);
  if (p.P <= 0) return SD_ERR_CUDA;
  const size_t need = ws_size(d);
  if (!ws || ws_bytes < need) return SD_ERR_WORKSPACE;
  const size_t slots = (size_t)p.B * p.Hkv + p.P;
  p.ws_o = reinterpret_cast<float *>(ws);
  p.ws_ml = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(ws) +
                                      round_up(slots * p.Mpad * p.D * 4, 256));
  CUtensorMap km, vm;
  const uint64_t rows = (uint64_t)p.num_blocks * p.Hkv * p.bs;
  p.kv3d = encode_tmap_kv_chunks_bf16(&km, k_cache, p.D, rows, kTile) &&
           encode_tmap_kv_chunks_bf16(&vm, v_cache, p.D, rows, kTile);
  if (!p.kv3d &&
      (!encode_tmap_2d_bf16(&km, k_cache, p.D, rows, (uint64_t)p.D * 2, 64, kTile) ||
       !encode_tmap_2d_bf16(&vm, v_cache, p.D, rows, (uint64_t)p.D * 2, 64, kTile)))
    return SD_ERR_CUDA;
  const bool window = p.window > 0 && p.window <= kWinMax && MT <= 2;
  if (!draft && window && MT == 1) {
    // cluster kernel with one query tile: it appends the new rows itself
    p.k_new = k_new;
    p.v_new = v_new;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
  } else if (!draft) {
    if (launch(append_kv_kernel<__nv_bfloat16>, dim3(p.B * p.n_q), dim3(256), 0, st, p,
               (const __nv_bfloat16 *)k_new, (const __nv_bfloat16 *)v_new,
               (__nv_bfloat16 *)k_cache, (__nv_bfloat16 *)v_cache) != cudaSuccess)
      return SD_ERR_CUDA;
  }
  if (window) {
    // every item reads at most window + n_q - 1 keys, over at most this many 16-key tiles
    const int tiles_max = (p.window + p.n_q - 1 + kTile - 1) / kTile + 1;
    return launch_window(p.D, MT, km, vm, p, tiles_max, st);
  }
  s = launch_bf16(p.D, rs, km, vm, p, st);
  if (s != SD_OK) return s;
  return cuda_status(
      combine_wide(p.B * p.Hkv * p.M, p.P, p.B * p.Hkv)
          ? launch(attn_combine_kernel<__nv_bfloat16, 4>, dim3(p.B * p.Hkv, p.M), dim3(512), 0,
                   st, p)
          : launch(attn_combine_kernel<__nv_bfloat16, 1>, dim3(p.B * p.Hkv, p.M), dim3(128), 0,
                   st, p));
}

}  // namespace attn
}  // namespace sdv

extern "C" {

size_t sd_verify_attn_workspace_size(const sd_attn_desc *desc) {
  if (sdv::attn::validate(desc, false) != SD_OK) return 0;
  return sdv::attn::ws_size(desc);
}

sd_status sd_verify_attn(const sd_attn_desc *desc, const void *q, const void *k_new,
                         const void *v_new, void *k_cache, void *v_cache,
                         const int32_t *block_table, const int32_t *ctx_len, void *out,
                         void *ws, size_t ws_bytes, sd_stream stream) {
  return sdv::attn::run(desc, false, q, k_new, v_new, k_cache, v_cache, block_table, ctx_len,
                        nullptr, out, ws, ws_bytes, (cudaStream_t)stream);
}

size_t sd_draft_xattn_workspace_size(const sd_attn_desc *desc) {
  if (sdv::attn::validate(desc, true) != SD_OK) return 0;
  return sdv::attn::ws_size(desc);
}

sd_status sd_draft_xattn(const sd_attn_desc *desc, const void *q, const void *k_cache,
                         const void *v_cache, const int32_t *block_table,
                         const int32_t *ctx_len, const int32_t *q_pos, void *out, void *ws,
                         size_t ws_bytes, sd_stream stream) {
  return sdv::attn::run(desc, true, q, nullptr, nullptr, const_cast<void *>(k_cache),
                        const_cast<void *>(v_cache), block_table, ctx_len, q_pos, out, ws,
                        ws_bytes, (cudaStream_t)stream);
}

}  // extern "C"
