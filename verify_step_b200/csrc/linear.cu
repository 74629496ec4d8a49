// Dense layers of the drafter and of the target: one projection of a few token rows against a
// bf16 weight matrix, with an RMSNorm / embedding-gather prologue and a store, residual-add or
// gated-GELU epilogue (sm_100a).
//
// "Gemma 4 MTP: drafter drafts, target verifies", section "drafter internal architecture": the
// drafter runs 4 transformer layers on the target's last-layer activation and its own token
// embedding, and the target runs its layers over the k+1 verified positions.  With m <= 64 token
// rows a projection reads each weight once and does 2m FLOPs with it: the weights' single pass
// through HBM bounds it, as it bounds the LM head.
//
// Two kernels per call (the first is skipped when the input is already bf16 rows that need no
// normalisation, gather or padding and no tickets are used: the product then reads x itself):
//  1. linear_stage_kernel: one CTA per token row gathers the row (the input columns and, for
//     the drafter's first projection, an embedding row chosen by token id), normalises it
//     (RMSNorm with gain) and writes it once as bf16 into the workspace, zero-padded to a
//     multiple of 64 columns (x'); it also clears the split tickets of kernel 2.
//  2. linear_umma_kernel<N>: the product on the tensor cores with the operands swapped so the
//     streamed weights are the MMA's M side, as in the dense LM head: A = a 128-row tile of W
//     [128 x 64] per pipeline stage, B = x' [N x 64] (N = m rounded up to 16, zero rows past m),
//     D = y^T tile [128 x N] float32 in tensor memory (two buffers).  Warp 0 issues the TMA
//     copies (no multicast; W evict-first, x' evict-last), warp 1 issues tcgen05.mma from one
//     thread, warps 2-5 read the accumulator (thread = output row).  Persistent: one CTA per
//     SM walks the work units (tile, K split); the K dimension is split so that the units
//     spread evenly over the SMs.  When every unit gets its own SM and a tile has 2, 4 or 8
//     splits, the splits are one thread-block cluster: each pushes its partial rows into the
//     shared memory of the CTA owning them and, after one cluster barrier, the owners add the
//     partials in split order and apply the epilogue.  Otherwise a split writes its [128 x m]
//     partial to the workspace and the last split of a tile to finish (atomic ticket, no
//     waiting) adds the partials in split order; either way the result does not depend on
//     the timing.
#include <algorithm>

#include "common.cuh"
#include "host.cuh"

namespace sdv {
namespace lin {

constexpr int BM = 128;      // weight rows per tile (UMMA M)
constexpr int BK = 64;       // K elements per stage (128-byte rows)
constexpr int kMaxM = 64;
constexpr int kMaxSplits = 32;
constexpr int kStageThreads = 256;

struct Params {
  // input rows
  int m, n, k, k64, k_x, x_f32;
  long long ld_x;
  const void *x;
  const __nv_bfloat16 *table;
  long long ld_table, table_rows, ld_tokens;
  const int32_t *tokens;
  const int32_t *token_sel;
  const float *gain;
  float eps;
  __nv_bfloat16 *norm_out;
  long long ld_norm_out;
  __nv_bfloat16 *xp;  // x' [m][k64] bf16 (workspace)
  // product
  int tiles, kblocks, splits, kb_per_split, units;
  int cluster;  // the splits of a tile are one thread-block cluster: partials summed via DSMEM
  int epi, out_f32;
  long long ld_out;
  void *out;
  float *part;              // [units][N][BM] partial sums (splits > 1)
  unsigned int *tickets;    // [tiles]
  int *status;
};

__device__ __forceinline__ float gelu_tanh(float z) {
  return 0.5f * z * (1.f + tanhf(0.7978845608028654f * (z + 0.044715f * z * z * z)));
}

__device__ __forceinline__ float4 bf16x4_to_f4(uint2 u) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

// Four consecutive input columns col .. col+3 of row r before normalisation (zeros for an
// invalid token).
__device__ __forceinline__ float4 input4(const Params &p, int r, int col, int tok) {
  if (col < p.k_x) {
    if (p.x_f32)
      return *reinterpret_cast<const float4 *>(static_cast<const float *>(p.x) + r * p.ld_x +
                                               col);
    return bf16x4_to_f4(*reinterpret_cast<const uint2 *>(
        static_cast<const __nv_bfloat16 *>(p.x) + r * p.ld_x + col));
  }
  if (tok < 0) return make_float4(0.f, 0.f, 0.f, 0.f);
  return bf16x4_to_f4(
      *reinterpret_cast<const uint2 *>(p.table + tok * p.ld_table + (col - p.k_x)));
}

// ------------------------------------------------------------------------------ staging

__global__ void __launch_bounds__(kStageThreads) linear_stage_kernel(const Params p) {
  __shared__ int s_tok;
  __shared__ float s_red[kStageThreads / 32];
  __shared__ float s_inv;
  pdl_trigger();  // the product kernel may start its weight copies meanwhile
  pdl_wait();
  const int r = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (r == 0 && p.splits > 1 && !p.cluster)
    for (int t = tid; t < p.tiles; t += blockDim.x) p.tickets[t] = 0u;
  if (tid == 0) {
    int t = -1;
    if (p.k_x < p.k) {
      int sel = 0;
      if (p.token_sel != nullptr) sel = p.token_sel[r];
      const long long span = p.ld_tokens > 0 ? p.ld_tokens : 1;
      if (sel >= 0 && sel < span) {
        t = p.tokens[r * p.ld_tokens + sel];
        if (t < 0 || t >= p.table_rows) t = -1;
      }
      if (t < 0) record_status(p.status, SD_ERR_DEVICE);
    }
    s_tok = t;
  }
  __syncthreads();
  const int tok = s_tok;
  float inv = 1.f;
  if (p.gain != nullptr) {
    float ss = 0.f;
    for (int c = tid * 4; c < p.k; c += kStageThreads * 4) {
      const float4 v = input4(p, r, c, tok);
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) s_red[warp] = ss;
    __syncthreads();
    if (tid == 0) {
      float t = 0.f;
      for (int w = 0; w < kStageThreads / 32; ++w) t += s_red[w];
      s_inv = rsqrtf(t / (float)p.k + p.eps);
    }
    __syncthreads();
    inv = s_inv;
  }
  for (int c = tid * 4; c < p.k64; c += kStageThreads * 4) {
    uint2 v2 = make_uint2(0u, 0u);
    if (c < p.k) {
      float4 x4 = input4(p, r, c, tok);
      if (p.gain != nullptr) {
        const float4 g = *reinterpret_cast<const float4 *>(p.gain + c);
        x4 = make_float4(x4.x * inv * g.x, x4.y * inv * g.y, x4.z * inv * g.z, x4.w * inv * g.w);
      }
      v2 = make_uint2(pack_bf16x2(x4.x, x4.y), pack_bf16x2(x4.z, x4.w));
      if (p.norm_out != nullptr)
        *reinterpret_cast<uint2 *>(p.norm_out + r * p.ld_norm_out + c) = v2;
    }
    *reinterpret_cast<uint2 *>(p.xp + (size_t)r * p.k64 + c) = v2;
  }
}

// ------------------------------------------------------------------------------ product

template <int N>
struct UCfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = N * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (192 * 1024 / STAGE_BYTES) < 8 ? (192 * 1024 / STAGE_BYTES) : 8;
  static constexpr uint32_t TMEM_COLS = (2 * N <= 32) ? 32 : (2 * N <= 64) ? 64 : 128;
  static constexpr int RECV_BYTES = BM * N * 4;  // partial rows pushed by the cluster's CTAs
  static constexpr size_t SMEM =
      1024 + (size_t)STAGES * STAGE_BYTES + RECV_BYTES + 8 * (2 * STAGES + 4) + 64;
  static constexpr int THREADS = 192;
};

// The epilogue of one output row i (this thread's) for token r: y = the row's product.  The
// gated form pairs row i (a gate row: i % 16 < 8) with row i + 8 of the same warp (lane + 8);
// every lane of the warp calls it for the same r.
__device__ __forceinline__ void apply_epilogue(const Params &p, int i, int r, float y, int lane,
                                               bool active = true) {
  if (p.epi == SD_EPI_GEGLU) {
    const float yu = __shfl_down_sync(0xffffffffu, y, 8);
    if (active && (lane & 8) == 0 && r < p.m) {
      const int f = (i >> 4) * 8 + (i & 7);
      if (f < p.n / 2)
        static_cast<__nv_bfloat16 *>(p.out)[r * p.ld_out + f] =
            __float2bfloat16_rn(gelu_tanh(y) * yu);
    }
    return;
  }
  if (!active || r >= p.m || i >= p.n) return;
  const long long o = r * p.ld_out + i;
  if (p.epi == SD_EPI_ADD)
    static_cast<float *>(p.out)[o] += y;
  else if (p.out_f32)
    static_cast<float *>(p.out)[o] = y;
  else
    static_cast<__nv_bfloat16 *>(p.out)[o] = __float2bfloat16_rn(y);
}

template <int N>
__global__ void __launch_bounds__(192, 1)
    linear_umma_kernel(const __grid_constant__ CUtensorMap wmap,
                       const __grid_constant__ CUtensorMap xmap, const Params p) {
  using C = UCfg<N>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *recv = reinterpret_cast<float *>(smem + (size_t)STAGES * C::STAGE_BYTES);  // [BM][N]
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)STAGES * C::STAGE_BYTES +
                                                C::RECV_BYTES);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;   // [2] accumulator ready
  uint64_t *tempty = tfull + 2;       // [2] accumulator drained
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *s_last = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // cluster mode: an arrival now, and a wait before the first distributed-shared-memory store,
  // so that no CTA writes into a peer that has not started
  if (p.cluster) cluster_arrive_relaxed();
  const uint32_t tmem_base = *tmem_slot;
  // x' and the tickets come from the staging kernel, which this kernel may overlap (it is
  // launched as its programmatic dependent): every role waits for it before touching global
  // memory, except that the producer first requests the weights of its first stages (the
  // weights are not written by the staging kernel)
  if (warp != 0) pdl_wait();

  if (warp == 0) {
    // ----------------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&wmap);
      tma_prefetch_desc(&xmap);
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_last();
      // the first STAGES stages (fresh barriers: no wait for a free stage): weights now,
      // x' rows once the staging kernel is done
      int pre_kb[STAGES];
      uint32_t pre = 0;
      for (int u = blockIdx.x; u < p.units && pre < (uint32_t)STAGES; u += gridDim.x) {
        const int tile = u / p.splits, split = u % p.splits;
        const int kb0 = split * p.kb_per_split;
        const int kb1 = min(p.kblocks, kb0 + p.kb_per_split);
        for (int kb = kb0; kb < kb1 && pre < (uint32_t)STAGES; ++kb, ++pre) {
          uint8_t *a = smem + (size_t)pre * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[pre], C::STAGE_BYTES);
          tma_load_2d_hint(a, &wmap, &full[pre], kb * BK, tile * BM, pol_w);
          pre_kb[pre] = kb;
        }
      }
      pdl_wait();
      for (uint32_t j = 0; j < pre; ++j)
        tma_load_2d_hint(smem + (size_t)j * C::STAGE_BYTES + C::A_BYTES, &xmap, &full[j],
                         pre_kb[j] * BK, 0, pol_x);
      uint32_t g = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        const int tile = u / p.splits, split = u % p.splits;
        const int kb0 = split * p.kb_per_split;
        const int kb1 = min(p.kblocks, kb0 + p.kb_per_split);
        for (int kb = kb0; kb < kb1; ++kb, ++g) {
          if (g < pre) continue;  // requested above
          const int stage = g % STAGES;
          const uint32_t ph = (g / STAGES) & 1;
          if (!mbar_wait(&empty[stage], ph ^ 1, abort_flag)) {
            record_status(p.status, SD_ERR_TIMEOUT);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t *a = smem + (size_t)stage * C::STAGE_BYTES;
          uint8_t *b = a + C::A_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d_hint(a, &wmap, &full[stage], kb * BK, tile * BM, pol_w);
          tma_load_2d_hint(b, &xmap, &full[stage], kb * BK, 0, pol_x);
        }
      }
      if (!ok) {
        for (uint32_t j = (g > (uint32_t)STAGES ? g - STAGES : 0); j < g; ++j)
          mbar_wait_timed(&full[j % STAGES], (j / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32(BM, N);
      uint32_t g = 0, i = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x, ++i) {
        const int split = u % p.splits;
        const int kb0 = split * p.kb_per_split;
        const int kb1 = min(p.kblocks, kb0 + p.kb_per_split);
        const uint32_t buf = i & 1, tph = (i >> 1) & 1;
        if (!mbar_wait(&tempty[buf], tph ^ 1, abort_flag)) {
          record_status(p.status, SD_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * N;
        for (int kb = kb0; kb < kb1; ++kb, ++g) {
          const int stage = g % STAGES;
          const uint32_t ph = (g / STAGES) & 1;
          if (!mbar_wait(&full[stage], ph, abort_flag)) {
            record_status(p.status, SD_ERR_TIMEOUT);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(smem + (size_t)stage * C::STAGE_BYTES);
          const uint32_t b = a + C::A_BYTES;
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks)
            umma_bf16(d_tmem, umma_desc_sw128(a + ks * 32), umma_desc_sw128(b + ks * 32), idesc,
                      (kb != kb0 || ks != 0) ? 1u : 0u);
          umma_commit(&empty[stage]);
        }
        if (ok) umma_commit(&tfull[buf]);
      }
    }
  } else {
    // ----------------------------------------------------------------------- epilogue
    // Every epilogue warp runs the same number of unit iterations and named barriers whatever
    // happens, so an abort cannot leave a warp waiting at a barrier: after a failed wait the
    // warp skips the work (later waits return at once) but keeps the barriers.
    const int quad = warp & 3;  // tensor-memory lanes 32*quad .. 32*quad+31
    const int row_in_tile = quad * 32 + lane;
    if (p.cluster) {
      // one unit per CTA; the tile's splits are the cluster's CTAs.  Each row of this split's
      // partial goes to the shared memory of the CTA owning the row (CTA r owns rows
      // [r BM/S, (r+1) BM/S)); the owners add them after the cluster barrier below.
      bool ok = *abort_flag == 0 && mbar_wait(&tfull[0], 0, abort_flag);
      if (!ok && *abort_flag == 0) {
        record_status(p.status, SD_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      tc_fence_after();
      float y[N];
      if (ok) {
        const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16);
#pragma unroll
        for (int c0 = 0; c0 < N; c0 += 16) {
          uint32_t rr[16];
          tmem_ld16(taddr + c0, rr);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) y[c0 + e] = __uint_as_float(rr[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < N; ++e) y[e] = 0.f;
      }
      tc_fence_before();
      mbar_arrive(&tempty[0]);
      cluster_wait();
      const uint32_t rank = cluster_ctarank();
      const int rows_per = BM / p.splits;
      const int owner = row_in_tile / rows_per;
      const uint32_t dst = dsmem_addr(
          smem_u32(recv + ((size_t)rank * rows_per + (row_in_tile - owner * rows_per)) * N),
          (uint32_t)owner);
#pragma unroll
      for (int r = 0; r < N; r += 4)
        st_dsmem_f4(dst + r * 4, make_float4(y[r], y[r + 1], y[r + 2], y[r + 3]));
    }
    uint32_t i = 0;
    for (int u = blockIdx.x; u < p.units && !p.cluster; u += gridDim.x, ++i) {
      const int tile = u / p.splits;
      const uint32_t buf = i & 1, tph = (i >> 1) & 1;
      bool ok = *abort_flag == 0 && mbar_wait(&tfull[buf], tph, abort_flag);
      if (!ok && *abort_flag == 0) {
        record_status(p.status, SD_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      tc_fence_after();
      const int row = tile * BM + row_in_tile;
      float y[N];
      if (ok) {
        const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + buf * N;
#pragma unroll
        for (int c0 = 0; c0 < N; c0 += 16) {
          uint32_t rr[16];
          tmem_ld16(taddr + c0, rr);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) y[c0 + e] = __uint_as_float(rr[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < N; ++e) y[e] = 0.f;
      }
      tc_fence_before();
      mbar_arrive(&tempty[buf]);
      if (p.splits == 1) {
        if (ok) {
#pragma unroll
          for (int r = 0; r < N; ++r) apply_epilogue(p, row, r, y[r], lane);
        }
        continue;
      }
      // ---- split K: partial to the workspace; the tile's last split reduces
      if (ok) {
        float *dst = p.part + (size_t)u * N * BM + row_in_tile;
#pragma unroll
        for (int r = 0; r < N; ++r)
          if (r < p.m) dst[(size_t)r * BM] = y[r];
        __threadfence();
      }
      named_barrier(1, 128);
      if (threadIdx.x == 64) {
        int last = 0;
        if (*abort_flag == 0) {
          const unsigned int t = atomicAdd(&p.tickets[tile], 1u);
          last = t == (unsigned int)(p.splits - 1);
        }
        *s_last = last;
      }
      named_barrier(1, 128);
      if (*s_last) {
        __threadfence();
        const int own = u % p.splits;
        const int s0 = u - own;  // first unit of the tile
        // partials added in split order; the loads of RB splits are issued together (this
        // split's own partial is still in registers)
        constexpr int RB = N <= 16 ? 8 : N <= 32 ? 4 : N <= 48 ? 2 : 1;
        float acc[N];
#pragma unroll
        for (int r = 0; r < N; ++r) acc[r] = 0.f;
        for (int sp0 = 0; sp0 < p.splits; sp0 += RB) {
          float v[RB][N];
#pragma unroll
          for (int q = 0; q < RB; ++q) {
            const int sp = sp0 + q;
            const bool load = sp < p.splits && sp != own;
            const float *src = p.part + (size_t)(s0 + sp) * N * BM + row_in_tile;
#pragma unroll
            for (int r = 0; r < N; ++r)
              v[q][r] = load && r < p.m ? __ldcg(src + (size_t)r * BM) : 0.f;
          }
#pragma unroll
          for (int q = 0; q < RB; ++q) {
            const int sp = sp0 + q;
            if (sp >= p.splits) break;
#pragma unroll
            for (int r = 0; r < N; ++r) acc[r] += sp == own ? y[r] : v[q][r];
          }
        }
#pragma unroll
        for (int r = 0; r < N; ++r) apply_epilogue(p, row, r, acc[r], lane);
        if (threadIdx.x == 64) p.tickets[tile] = 0u;
      }
    }
  }
  if (p.cluster) {
    // every CTA of the cluster reaches this barrier once (no role returns early), so all partial
    // rows have landed in their owners after it; each owner adds its rows' S partials in split
    // order and applies the epilogue
    if (warp < 2) cluster_wait();  // the first phase (the epilogue warps waited before storing)
    cluster_sync();
    if (warp >= 2) {
      const int quad = warp & 3;
      const int row_in_tile = quad * 32 + lane;
      const int rank = (int)cluster_ctarank();
      const int rows_per = BM / p.splits;
      const bool mine = row_in_tile / rows_per == rank;
      const int tile = blockIdx.x / p.splits;
      float acc[N];
#pragma unroll
      for (int r = 0; r < N; ++r) acc[r] = 0.f;
      if (mine) {
        for (int sp = 0; sp < p.splits; ++sp) {
          const float4 *src = reinterpret_cast<const float4 *>(
              recv + ((size_t)sp * rows_per + (row_in_tile - rank * rows_per)) * N);
#pragma unroll
          for (int r = 0; r < N; r += 4) {
            const float4 v = src[r / 4];
            acc[r] += v.x;
            acc[r + 1] += v.y;
            acc[r + 2] += v.z;
            acc[r + 3] += v.w;
          }
        }
      }
#pragma unroll
      for (int r = 0; r < N; ++r) apply_epilogue(p, tile * BM + row_in_tile, r, acc[r], lane, mine);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    if (*abort_flag) {
      // let MMAs already issued drain before the tensor memory is released
      const unsigned long long t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 1000000ull) {
      }
    }
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------ host side

struct Shape {
  int N, tiles, kblocks, splits, kb_per_split, units, grid;
  bool cluster;
};

static int n_of(int m) { return m <= 16 ? 16 : m <= 32 ? 32 : m <= 48 ? 48 : 64; }

// Work split of a call: S splits of the K blocks per 128-row tile, chosen to minimise a time
// model of the busiest SM: ceil(tiles S / SMs) units, each its K blocks at about 0.36 us (16 KB
// of weights and 4 KB of x' at a fair share of the HBM rate) plus, when split, about 2 us of
// partial write, fence and ticket; and the reductions the SM finishes (ceil(tiles / SMs) tiles,
// about 0.5 us per split read back).  (At 24 rows, d 5376: the gated MLP's 336 tiles take 2
// splits, 87.9 us against 94.7 unsplit.)
// Clusters of S CTAs of the product kernel for N that fit on the device at once (0 where the
// device cannot say, e.g. without a GPU).
static int max_clusters(int N, int S);

static Shape shape_of(int m, int n, int k, bool allow_cluster = false) {
  Shape s;
  s.N = n_of(m);
  s.tiles = (n + BM - 1) / BM;
  s.kblocks = (k + BK - 1) / BK;
  const int sms = std::max(sm_count(), 1);
  double best = -1.0;
  int best_s = 1;
  for (int S = 1; S <= std::min(kMaxSplits, s.kblocks); ++S) {
    const int kps = (s.kblocks + S - 1) / S;
    const int S_eff = (s.kblocks + kps - 1) / kps;  // every split non-empty
    if (S_eff != S) continue;
    const long long units = (long long)s.tiles * S;
    const double per_unit = kps * 0.36 + (S > 1 ? 2.0 : 0.0);
    double cost = (double)((units + sms - 1) / sms) * per_unit;
    if (S > 1) cost += (double)((s.tiles + sms - 1) / sms) * 0.5 * S;
    if (best < 0.0 || cost < best) {
      best = cost;
      best_s = S;
    }
  }
  // the splits of a tile as one cluster (2, 4 or 8 CTAs, whole 16-row blocks per owner) when
  // every unit gets its own SM: partials summed through distributed shared memory, about
  // 0.8 us, no workspace round trip or ticket
  bool cluster = false;
  for (int S = 2; S <= 8 && allow_cluster; S *= 2) {
    if (S > s.kblocks || (long long)s.tiles * S > sms || s.tiles > max_clusters(s.N, S)) break;
    const int kps = (s.kblocks + S - 1) / S;
    if ((s.kblocks + kps - 1) / kps != S) continue;
    const double cost = kps * 0.36 + 0.8;
    if (cost < best) {
      best = cost;
      best_s = S;
      cluster = true;
    }
  }
  s.splits = best_s;
  s.cluster = cluster;
  s.kb_per_split = (s.kblocks + best_s - 1) / best_s;
  s.units = s.tiles * best_s;
  s.grid = cluster ? s.units : std::min(s.units, sms);
  return s;
}

struct Layout {
  size_t xp, part, tickets, total;
};

static Layout layout_of(const sd_linear_desc *d, const Shape &s) {
  Layout l;
  const size_t k64 = (size_t)s.kblocks * BK;
  l.xp = 0;
  l.part = round_up((size_t)d->m * k64 * 2, 256);
  const size_t part_bytes = s.splits > 1 && !s.cluster ? (size_t)s.units * s.N * BM * 4 : 0;
  l.tickets = l.part + round_up(part_bytes, 256);
  l.total = l.tickets + round_up((size_t)s.tiles * 4, 256);
  return l;
}

static sd_status validate(const sd_linear_desc *d, const void *x, const void *W, void *out,
                          const void *table, const int32_t *tokens) {
  if (!d) return SD_ERR_INVALID_ARG;
  if (d->m < 0 || d->n < 1 || d->k < 1 || d->k_gather < 0 || d->k_gather > d->k)
    return SD_ERR_INVALID_ARG;
  if (d->m == 0) return SD_OK;
  if (!W || !out || (d->k_gather < d->k && !x)) return SD_ERR_INVALID_ARG;
  if (d->x_dtype != SD_F32 && d->x_dtype != SD_BF16) return SD_ERR_INVALID_ARG;
  if (d->epilogue != SD_EPI_STORE && d->epilogue != SD_EPI_ADD && d->epilogue != SD_EPI_GEGLU)
    return SD_ERR_INVALID_ARG;
  if (d->out_dtype != SD_F32 && d->out_dtype != SD_BF16) return SD_ERR_INVALID_ARG;
  if (d->epilogue == SD_EPI_ADD && d->out_dtype != SD_F32) return SD_ERR_INVALID_ARG;
  if (d->epilogue == SD_EPI_GEGLU && d->out_dtype != SD_BF16) return SD_ERR_INVALID_ARG;
  if (d->norm_out && !d->norm_gain) return SD_ERR_INVALID_ARG;
  if (d->m > kMaxM || d->n % 16 != 0 || d->k % 32 != 0 || d->k_gather % 8 != 0)
    return SD_ERR_UNSUPPORTED;
  const int k_x = d->k - d->k_gather;
  if (k_x > 0 && (d->ld_x < k_x || d->ld_x % 4 != 0 || !aligned16(x))) return SD_ERR_INVALID_ARG;
  if (d->k_gather > 0) {
    if (!table || !tokens || d->table_rows < 1 || d->ld_table < d->k_gather ||
        d->ld_table % 4 != 0 || !aligned16(table) || d->ld_tokens < 0)
      return SD_ERR_INVALID_ARG;
  }
  if (!aligned16(W) || (d->norm_gain && !aligned16(d->norm_gain))) return SD_ERR_INVALID_ARG;
  const int out_cols = d->epilogue == SD_EPI_GEGLU ? d->n / 2 : d->n;
  if (d->ld_out < out_cols) return SD_ERR_INVALID_ARG;
  if (d->norm_out && (d->ld_norm_out < d->k || d->ld_norm_out % 4 != 0 ||
                      (reinterpret_cast<uintptr_t>(d->norm_out) & 7u) != 0))
    return SD_ERR_INVALID_ARG;
  return SD_OK;
}

// The product is launched as a programmatic dependent of the staging kernel (always: the two
// are one call), so its launch, set-up and first weight copies overlap the staging.
template <int N>
static sd_status launch_product(const CUtensorMap &wm, const CUtensorMap &xm, const Params &p,
                                int grid, int cluster, cudaStream_t st) {
  using C = UCfg<N>;
  static int configured[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64 || configured[dev] != dev + 1) {
    if (cudaFuncSetAttribute(linear_umma_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)C::SMEM) != cudaSuccess)
      return SD_ERR_CUDA;
    if (dev < 64) configured[dev] = dev + 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster > 1 ? cluster : 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster > 1 ? 2 : 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, linear_umma_kernel<N>, wm, xm, p));
}

template <int N>
static int max_clusters_n(int S) {
  using C = UCfg<N>;
  if (cudaFuncSetAttribute(linear_umma_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)C::SMEM) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cudaLaunchAttribute a[1];
  a[0].id = cudaLaunchAttributeClusterDimension;
  a[0].val.clusterDim.x = S;
  a[0].val.clusterDim.y = 1;
  a[0].val.clusterDim.z = 1;
  cfg.attrs = a;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, linear_umma_kernel<N>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  return n;
}

static int max_clusters(int N, int S) {
  static int cache[64][4][4];  // [device][N / 16 - 1][log2 S - 1] = value + 1
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  const int ni = N / 16 - 1, si = S == 2 ? 0 : S == 4 ? 1 : 2;
  if (dev < 64 && cache[dev][ni][si] > 0) return cache[dev][ni][si] - 1;
  int v = 0;
  switch (N) {
    case 16: v = max_clusters_n<16>(S); break;
    case 32: v = max_clusters_n<32>(S); break;
    case 48: v = max_clusters_n<48>(S); break;
    default: v = max_clusters_n<64>(S); break;
  }
  if (dev < 64) cache[dev][ni][si] = v + 1;
  return v;
}

}  // namespace lin
}  // namespace sdv

extern "C" size_t sd_linear_workspace_size(const sd_linear_desc *d) {
  using namespace sdv::lin;
  if (!d || d->m < 1 || d->m > kMaxM || d->n < 1 || d->n % 16 || d->k < 1 || d->k % 32)
    return 0;
  return layout_of(d, shape_of(d->m, d->n, d->k)).total;
}

extern "C" sd_status sd_linear(const sd_linear_desc *d, const void *x, const void *W, void *out,
                               const void *table, const int32_t *tokens,
                               const int32_t *token_sel, sd_stream stream) {
  using namespace sdv;
  using namespace sdv::lin;
  sd_status s = validate(d, x, W, out, table, tokens);
  if (s != SD_OK || d->m == 0) return s;
  // the workspace is laid out for the plan without clusters (the larger one), so its size
  // does not depend on what the device reports
  const Shape sh = shape_of(d->m, d->n, d->k, true);
  const Layout lay = layout_of(d, shape_of(d->m, d->n, d->k));
  if (!d->ws || d->ws_bytes < lay.total || !aligned16(d->ws)) return SD_ERR_WORKSPACE;
  uint8_t *ws = static_cast<uint8_t *>(d->ws);

  Params p{};
  p.m = d->m;
  p.n = d->n;
  p.k = d->k;
  p.k64 = sh.kblocks * BK;
  p.k_x = d->k - d->k_gather;
  p.x_f32 = d->x_dtype == SD_F32;
  p.ld_x = d->ld_x;
  p.x = x;
  p.table = static_cast<const __nv_bfloat16 *>(table);
  p.ld_table = d->ld_table;
  p.table_rows = d->table_rows;
  p.ld_tokens = d->ld_tokens;
  p.tokens = tokens;
  p.token_sel = token_sel;
  p.gain = d->norm_gain;
  p.eps = d->norm_eps;
  p.norm_out = static_cast<__nv_bfloat16 *>(d->norm_out);
  p.ld_norm_out = d->ld_norm_out;
  p.xp = reinterpret_cast<__nv_bfloat16 *>(ws + lay.xp);
  p.tiles = sh.tiles;
  p.kblocks = sh.kblocks;
  p.splits = sh.splits;
  p.kb_per_split = sh.kb_per_split;
  p.units = sh.units;
  p.cluster = sh.cluster ? 1 : 0;
  p.epi = d->epilogue;
  p.out_f32 = d->out_dtype == SD_F32;
  p.ld_out = d->ld_out;
  p.out = out;
  p.part = reinterpret_cast<float *>(ws + lay.part);
  p.tickets = reinterpret_cast<unsigned int *>(ws + lay.tickets);
  p.status = device_status_word();

  // weights: [128 rows x 64 columns] boxes, 128-byte swizzle (rows past n and columns past k
  // arrive as zeros); x': [N rows x 64 columns] boxes of the m staged rows (rows past m zero)
  // A bf16 input that needs no normalisation, gather or padding (and no split tickets to
  // clear) is read by the product directly: no staging kernel
  const bool direct = d->x_dtype == SD_BF16 && !d->norm_gain && d->k_gather == 0 &&
                      d->k % BK == 0 && d->ld_x % 8 == 0 && !d->norm_out &&
                      (sh.cluster || sh.splits == 1);
  CUtensorMap wm, xm;
  const bool xok =
      direct ? encode_tmap_2d_bf16(&xm, x, (uint64_t)d->k, (uint64_t)d->m,
                                   (uint64_t)d->ld_x * 2, BK, (uint32_t)sh.N)
             : encode_tmap_2d_bf16(&xm, p.xp, (uint64_t)p.k64, (uint64_t)d->m,
                                   (uint64_t)p.k64 * 2, BK, (uint32_t)sh.N);
  if (!encode_tmap_2d_bf16(&wm, W, (uint64_t)d->k, (uint64_t)d->n, (uint64_t)d->k * 2, BK, BM) ||
      !xok)
    return SD_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  if (!direct &&
      launch(linear_stage_kernel, dim3(d->m), dim3(kStageThreads), 0, st, p) != cudaSuccess)
    return SD_ERR_CUDA;
  const int cl = sh.cluster ? sh.splits : 1;
  switch (sh.N) {
    case 16: return launch_product<16>(wm, xm, p, sh.grid, cl, st);
    case 32: return launch_product<32>(wm, xm, p, sh.grid, cl, st);
    case 48: return launch_product<48>(wm, xm, p, sh.grid, cl, st);
    default: return launch_product<64>(wm, xm, p, sh.grid, cl, st);
  }
}
