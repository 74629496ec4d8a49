// LM head over the vocabulary, dense and clustered (sm_100a).
//
// Dense: logits[i, v] = h[i] . W[v] for a 262144-token vocabulary (Gemma 4 MTP serving guide,
// section 1; GeekNews summary of the Google blog, section "MTP drafter internal optimisations":
// the final logit projection is a major cost).  With m = B * (k+1) rows of h (24 at B = 8,
// k = 2) the product is a weight stream: W is read once, 2.8 GB at d = 5376.
//
// bf16 design (tcgen05): swap A and B so the streamed operand is the MMA's M side.
//   A = a 128-row vocab tile of W [128 x 64] per pipeline stage (K-major, 128-byte swizzle),
//   B = h [N x 64] (N = m rounded up to the instruction's N, zero rows past m),
//   D = logits^T tile [128 x N] float32 in tensor memory (two buffers, so the epilogue of
//   one tile overlaps the MMAs of the next).
//   Warp 0 issues TMA loads (cp.async.bulk.tensor, no multicast; W evict-first, h
//   evict-last in L2), warp 1 allocates tensor memory and issues tcgen05.mma from one thread,
//   warps 2-5 read the accumulator with tcgen05.ld (thread = vocab row) and store
//   logits[i, v] coalesced along v.  Persistent: one CTA per SM walks vocab tiles.
//
// Clustered (drafter side; the pages give no algorithm, this is one flat level): centroid
// scores with the same kernel, per-row top-c selection, -inf fill, exact logits of the kept
// clusters' tokens gathered from cluster-major weights.
//
// float32 dense path: one warp per vocab row, plain FMA.
#include <cfloat>

#include "common.cuh"
#include "host.cuh"

namespace sdv {
namespace head {

constexpr int BM = 128;  // vocab rows per tile (UMMA M)
constexpr int BK = 64;   // K elements per stage (128-byte rows)

struct Params {
  int M, d, V, ld;
  int num_tiles, kblocks;
  float *logits;
  int *status;
};

template <int N>
struct UCfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = N * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (200 * 1024 / STAGE_BYTES) < 8 ? (200 * 1024 / STAGE_BYTES) : 8;
  static constexpr uint32_t TMEM_COLS = (2 * N <= 32) ? 32 : (2 * N <= 64) ? 64
                                      : (2 * N <= 128) ? 128 : (2 * N <= 256) ? 256 : 512;
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 8 * (2 * STAGES + 4) + 64;
  static constexpr int THREADS = 192;
};

template <int N>
__global__ void __launch_bounds__(192, 1)
    lm_head_umma_kernel(const __grid_constant__ CUtensorMap wmap,
                        const __grid_constant__ CUtensorMap hmap, const Params p) {
  using C = UCfg<N>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)STAGES * C::STAGE_BYTES);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;   // [2] accumulator ready
  uint64_t *tempty = tfull + 2;       // [2] accumulator drained
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

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
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // h (and the logits buffer) may come from earlier kernels

  if (warp == 0) {
    // ----------------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&wmap);
      tma_prefetch_desc(&hmap);
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_h = l2_policy_evict_last();
      uint32_t g = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        for (int kb = 0; kb < p.kblocks; ++kb, ++g) {
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
          tma_load_2d_hint(b, &hmap, &full[stage], kb * BK, 0, pol_h);
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
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++i) {
        const uint32_t buf = i & 1, tph = (i >> 1) & 1;
        if (!mbar_wait(&tempty[buf], tph ^ 1, abort_flag)) {
          record_status(p.status, SD_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * N;
        for (int kb = 0; kb < p.kblocks; ++kb, ++g) {
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
                      (kb | ks) != 0);
          umma_commit(&empty[stage]);
        }
        if (ok) umma_commit(&tfull[buf]);
      }
    }
  } else {
    // ----------------------------------------------------------------------- epilogue
    const int quad = warp & 3;  // tensor-memory lanes 32*quad .. 32*quad+31
    uint32_t i = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++i) {
      const uint32_t buf = i & 1, tph = (i >> 1) & 1;
      if (!mbar_wait(&tfull[buf], tph, abort_flag)) {
        record_status(p.status, SD_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int v = tile * BM + quad * 32 + lane;
      const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + buf * N;
#pragma unroll
      for (int c0 = 0; c0 < N; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(taddr + c0, r);
        tmem_ld_wait();
        if (v < p.V) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int m = c0 + e;
            if (m < p.M) p.logits[(size_t)m * p.ld + v] = __uint_as_float(r[e]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[buf]);
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

// float32: one warp per (vocab row); all m rows.
__global__ void lm_head_f32_kernel(const float *h, const float *w, const Params p) {
  pdl_wait();
  const int v = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (v >= p.V) return;
  const float *wr = w + (size_t)v * p.d;
  for (int m = 0; m < p.M; ++m) {
    const float *hr = h + (size_t)m * p.d;
    float acc = 0.f;
    for (int c = lane; c < p.d; c += 32) acc = fmaf(hr[c], wr[c], acc);
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) p.logits[(size_t)m * p.ld + v] = acc;
  }
}

// Per row m (blockIdx.y): block 0 selects the top_c clusters by score (ties -> lower id) and
// writes them in ascending id order; blocks 1.. write -inf over the row's logits meanwhile
// (the kept clusters' tokens are overwritten by the next kernel).
//
// Selection: an exact radix select over 32-bit keys ordered by descending score (smaller key =
// higher score; -0.0 and +0.0 are one key), most significant byte first, finds the key T of
// the top_c-th best cluster and how many clusters with key T are kept; the kept set is then
// read out in id order with two block scans (ties at T go to the lowest ids).
constexpr int kSelThreads = 256;

__device__ __forceinline__ uint32_t desc_key(float score) {
  uint32_t u = __float_as_uint(score == 0.f ? 0.f : score);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // ascending order of floats
  return ~u;
}

// Exclusive prefix sum of v over the block (kSelThreads threads); also returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int *s_warp, int &total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  int base = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < kSelThreads / 32; ++w) {
    const int t = s_warp[w];
    base += w < warp ? t : 0;
    total += t;
  }
  __syncthreads();
  return base + x - v;
}

__global__ void __launch_bounds__(kSelThreads) select_fill_kernel(const float *scores, int C,
                                                                  int top_c, int32_t *sel,
                                                                  float *logits, int V, int ld,
                                                                  int vec4) {
  extern __shared__ uint32_t skey[];  // [C]
  __shared__ int hist[256];
  __shared__ int s_warp[kSelThreads / 32];
  __shared__ int s_digit, s_before;
  pdl_wait();
  const int m = blockIdx.y;
  if (blockIdx.x > 0) {
    float *row = logits + (size_t)m * ld;
    const int nb = gridDim.x - 1, bx = blockIdx.x - 1;
    if (vec4) {
      float4 *r4 = reinterpret_cast<float4 *>(row);
      const float4 ninf = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      for (int i = bx * kSelThreads + threadIdx.x; i < V / 4; i += nb * kSelThreads) r4[i] = ninf;
    } else {
      for (int i = bx * kSelThreads + threadIdx.x; i < V; i += nb * kSelThreads)
        row[i] = -INFINITY;
    }
    return;
  }
  const int tid = threadIdx.x, lane = tid & 31;
  for (int i = tid; i < C; i += kSelThreads) skey[i] = desc_key(scores[(size_t)m * C + i]);
  uint32_t prefix = 0, mask = 0;
  int need = top_c;  // clusters still to take among the keys matching prefix under mask
  for (int shift = 24; shift >= 0; shift -= 8) {
    hist[tid] = 0;  // kSelThreads == 256 bins
    __syncthreads();
    for (int i = tid; i < C; i += kSelThreads) {
      const uint32_t k = skey[i];
      if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255], 1);
    }
    __syncthreads();
    if (tid < 32) {
      // lane owns digits [8 lane, 8 lane + 8): find the digit where the count reaches need
      int cnt[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = hist[lane * 8 + j];
        sum += cnt[j];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int run = incl - sum;  // keys with a smaller digit in lower lanes
      const unsigned hit = __ballot_sync(0xffffffffu, run < need && need <= incl);
      if (lane == __ffs(hit) - 1) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run < need && need <= run + cnt[j]) {
            s_digit = lane * 8 + j;
            s_before = run;
          }
          run += cnt[j];
        }
      }
    }
    __syncthreads();
    prefix |= (uint32_t)s_digit << shift;
    mask |= 255u << shift;
    need -= s_before;
    __syncthreads();
  }
  // prefix is the key T of the top_c-th cluster; every key < T is kept, and the `need` keys
  // equal to T with the lowest ids.  Thread tid reads ids [tid * per, tid * per + per).
  const int per = (C + kSelThreads - 1) / kSelThreads;
  const int i0 = tid * per, i1 = min(C, i0 + per);
  int ties = 0;
  for (int i = i0; i < i1; ++i) ties += skey[i] == prefix;
  int total;
  int tie_rank = block_exclusive_scan(ties, s_warp, total);
  int takes = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t k = skey[i];
    takes += k < prefix || (k == prefix && tie_rank++ < need);
  }
  int out = block_exclusive_scan(takes, s_warp, total);
  tie_rank -= ties;  // back to this thread's first tie
  for (int i = i0; i < i1; ++i) {
    const uint32_t k = skey[i];
    if (k < prefix || (k == prefix && tie_rank++ < need)) sel[(size_t)m * top_c + out++] = i;
  }
  (void)lane;
}

// Exact logits of the kept clusters' tokens.  The work is M * top_c * ceil(cs / TK) units of TK
// tokens; a persistent grid of warps takes contiguous ranges of units, so consecutive units of
// a warp almost always share the row m.  Lane l multiplies elements l*8 + q*256 + [0, 8) of a
// weight row and keeps those hidden values in registers (reloaded only when m changes); the
// weight loads of a unit's TK tokens are all in flight before the dot products (d <= 256 * KMAX).
template <int KMAX, int TK>
__global__ void __launch_bounds__(256) cluster_logits_kernel(
    const __nv_bfloat16 *h, const __nv_bfloat16 *w_cm, const int32_t *cluster_tokens,
    const int32_t *sel, int M, int top_c, int cs, int d, int C, int V, int ld, float *logits,
    int *status) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const long long n_warps = (long long)gridDim.x * (blockDim.x >> 5);
  const long long wid = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int upc = (cs + TK - 1) / TK;  // units per (row, cluster)
  const long long U = (long long)M * top_c * upc;
  const long long u_begin = U * wid / n_warps, u_end = U * (wid + 1) / n_warps;
  const int nk = (d + 255) / 256;
  float hr[KMAX][8];
  int m_loaded = -1;
  for (long long u = u_begin; u < u_end; ++u) {
    const int ms = (int)(u / upc);
    const int t0 = (int)(u % upc) * TK;
    const int m = ms / top_c, slot = ms % top_c;
    const int c = sel[(size_t)m * top_c + slot];
    if (c < 0 || c >= C) {
      if (lane == 0) record_status(status, SD_ERR_DEVICE);
      continue;
    }
    uint4 raw[TK][KMAX];
#pragma unroll
    for (int t = 0; t < TK; ++t)
#pragma unroll
      for (int q = 0; q < KMAX; ++q) {
        const int k0 = lane * 8 + q * 256;
        raw[t][q] = (q < nk && k0 < d && t0 + t < cs)
                        ? __ldg(reinterpret_cast<const uint4 *>(
                              w_cm + ((size_t)c * cs + t0 + t) * d + k0))
                        : make_uint4(0, 0, 0, 0);
      }
    if (m != m_loaded) {
#pragma unroll
      for (int q = 0; q < KMAX; ++q) {
        const int k0 = lane * 8 + q * 256;
        uint4 hv = make_uint4(0, 0, 0, 0);
        if (q < nk && k0 < d) hv = __ldg(reinterpret_cast<const uint4 *>(h + (size_t)m * d + k0));
        const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&hv);
#pragma unroll
        for (int r = 0; r < 8; ++r) hr[q][r] = __bfloat162float(e[r]);
      }
      m_loaded = m;
    }
    float acc[TK];
#pragma unroll
    for (int t = 0; t < TK; ++t) {
      acc[t] = 0.f;
#pragma unroll
      for (int q = 0; q < KMAX; ++q) {
        const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&raw[t][q]);
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[t] = fmaf(__bfloat162float(e[r]), hr[q][r], acc[t]);
      }
    }
#pragma unroll
    for (int t = 0; t < TK; ++t)
      for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
    if (lane < TK && t0 + lane < cs) {
      float mine = acc[0];
#pragma unroll
      for (int t = 1; t < TK; ++t)
        if (lane == t) mine = acc[t];
      const int tok = cluster_tokens[(size_t)c * cs + t0 + lane];
      if (tok < 0 || tok >= V)
        record_status(status, SD_ERR_DEVICE);
      else
        logits[(size_t)m * ld + tok] = mine;
    }
  }
}

// Same logits with the weights staged by bulk copies (d <= 1024, cluster_size a multiple of
// kClTok): the work is M * top_c * cs / kClTok units of kClTok tokens, each unit's weights one
// contiguous block of the cluster-major matrix.  A persistent CTA per SM takes a contiguous
// range of units; its producer warp streams them (weights and token ids, cp.async.bulk) through
// a kClStages-deep mbarrier ring, and each of the kClWarps consumer warps takes one token of a
// unit: lane l multiplies elements l*8 + q*256 + [0, 8) of the staged row with the hidden
// values it keeps in registers (reloaded when the row m changes), in two accumulator chains.
constexpr int kClTok = 16;
constexpr int kClStages = 6;
constexpr int kClWarps = kClTok;  // one token per warp: 17 warps per SM hide the latency
constexpr int kClUnitBytes = kClTok * 1024 * 2;  // largest unit (d = 1024)
constexpr size_t kClSmem = 128 + (size_t)kClStages * kClUnitBytes + kClStages * kClTok * 4 +
                           kClStages * 16 + kClStages * 16 + 16;

__global__ void __launch_bounds__(32 * (kClWarps + 1), 1) cluster_logits_tma_kernel(
    const __nv_bfloat16 *h, const __nv_bfloat16 *w_cm, const int32_t *cluster_tokens,
    const int32_t *sel, int M, int top_c, int cs, int d, int C, int V, int ld, float *logits,
    int *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint8_t *stages = smem;  // [kClStages][kClTok * d * 2]
  int32_t *tok = reinterpret_cast<int32_t *>(stages + (size_t)kClStages * kClUnitBytes);
  int4 *rec = reinterpret_cast<int4 *>(tok + kClStages * kClTok);  // (m, c, t0, tokens)
  uint64_t *full = reinterpret_cast<uint64_t *>(rec + kClStages);
  uint64_t *empty = full + kClStages;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + kClStages);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  if (threadIdx.x < 2 * kClStages) {
    mbar_init(&full[threadIdx.x], threadIdx.x < kClStages ? 1u : (uint32_t)kClWarps);
    fence_mbar_init();
  }
  if (threadIdx.x == 0) *abort_flag = 0;
  __syncthreads();
  const int upc = cs / kClTok;  // units per (row, cluster)
  const long long U = (long long)M * top_c * upc;
  const long long u0 = U * blockIdx.x / gridDim.x, u1 = U * (blockIdx.x + 1) / gridDim.x;
  const uint32_t wbytes = (uint32_t)kClTok * d * 2;

  if (warp == kClWarps) {
    // ------------------------------------------------------------------- producer warp
    if (lane != 0) return;
    long long u = u0;
    for (; u < u1; ++u) {
      const int it = (int)(u - u0), stg = it % kClStages;
      if (!mbar_wait(&empty[stg], ((it / kClStages) & 1) ^ 1, abort_flag)) {
        record_status(status, SD_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      const int ms = (int)(u / upc), t0 = (int)(u % upc) * kClTok;
      const int m = ms / top_c, slot = ms % top_c;
      const int c = sel[(size_t)m * top_c + slot];
      if (c < 0 || c >= C) {
        record_status(status, SD_ERR_DEVICE);
        rec[stg] = make_int4(m, c, t0, 0);
        mbar_arrive(&full[stg]);
        continue;
      }
      rec[stg] = make_int4(m, c, t0, kClTok);
      mbar_arrive_expect_tx(&full[stg], wbytes + kClTok * 4);
      bulk_load(stages + (size_t)stg * kClUnitBytes, w_cm + ((size_t)c * cs + t0) * d, wbytes,
                &full[stg]);
      bulk_load(tok + stg * kClTok, cluster_tokens + (size_t)c * cs + t0, kClTok * 4,
                &full[stg]);
    }
    if (*abort_flag) {
      // wait (bounded) for the copies this CTA issued before leaving
      const long long n = u - u0;
      for (long long j = (n > kClStages ? n - kClStages : 0); j < n; ++j)
        mbar_wait_timed(&full[j % kClStages], (uint32_t)((j / kClStages) & 1));
    }
    return;
  }

  // --------------------------------------------------------------------- consumer warps
  const int nk = d / 256 + (d % 256 != 0);
  float hr[4][8];
  int m_loaded = -1;
  for (long long u = u0; u < u1; ++u) {
    const int it = (int)(u - u0), stg = it % kClStages;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[stg], (it / kClStages) & 1, abort_flag))) {
      record_status(status, SD_ERR_TIMEOUT);
      *abort_flag = 1;
      break;
    }
    const int4 r = rec[stg];
    if (r.w > 0) {
      if (r.x != m_loaded) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int k0 = lane * 8 + q * 256;
          uint4 hv = make_uint4(0, 0, 0, 0);
          if (q < nk && k0 < d)
            hv = __ldg(reinterpret_cast<const uint4 *>(h + (size_t)r.x * d + k0));
          const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&hv);
#pragma unroll
          for (int j = 0; j < 8; ++j) hr[q][j] = __bfloat162float(e[j]);
        }
        m_loaded = r.x;
      }
      const uint8_t *row = stages + (size_t)stg * kClUnitBytes + (size_t)warp * d * 2;
      float acc2[2] = {0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int k0 = lane * 8 + q * 256;
        if (q < nk && k0 < d) {
          const uint4 raw = *reinterpret_cast<const uint4 *>(row + (size_t)k0 * 2);
          const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&raw);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            acc2[j & 1] = fmaf(__bfloat162float(e[j]), hr[q][j], acc2[j & 1]);
        }
      }
      float acc = acc2[0] + acc2[1];
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) {
        const int id = tok[stg * kClTok + warp];
        if (id < 0 || id >= V)
          record_status(status, SD_ERR_DEVICE);
        else
          logits[(size_t)r.x * ld + id] = acc;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stg]);
  }
}

// Centroid scores of the clustered head, score[i, c] = h[i] . centroid[c], for up to 16 rows:
// one warp per centroid (its row read once, 16-byte loads), the rows of h in shared memory.
// A GEMV this small (2 MB of centroids) needs many CTAs in flight rather than tensor cores.
__global__ void __launch_bounds__(256) centroid_scores_kernel(const __nv_bfloat16 *h,
                                                              const __nv_bfloat16 *cent, int M,
                                                              int d, int C, float *scores) {
  extern __shared__ float hs[];  // [M][d]
  pdl_trigger();
  pdl_wait();
  for (int i = threadIdx.x; i < M * d / 8; i += blockDim.x) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(h) + i);
    const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&raw);
#pragma unroll
    for (int r = 0; r < 8; ++r) hs[i * 8 + r] = __bfloat162float(e[r]);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x * (blockDim.x >> 5) + warp;
  // this lane's part of the centroid row, loaded before the rows of h are needed (d <= 1024)
  uint4 raw[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int k0 = lane * 8 + q * 256;
    raw[q] = (c < C && k0 < d) ? __ldg(reinterpret_cast<const uint4 *>(cent + (size_t)c * d + k0))
                               : make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  if (c >= C) return;
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int k0 = lane * 8 + q * 256;
    if (k0 >= d) break;
    const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&raw[q]);
    float w[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) w[r] = __bfloat162float(e[r]);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i < M) {
        const float4 a = *reinterpret_cast<const float4 *>(hs + i * d + k0);
        const float4 b = *reinterpret_cast<const float4 *>(hs + i * d + k0 + 4);
        acc[i] = fmaf(w[0], a.x, acc[i]);
        acc[i] = fmaf(w[1], a.y, acc[i]);
        acc[i] = fmaf(w[2], a.z, acc[i]);
        acc[i] = fmaf(w[3], a.w, acc[i]);
        acc[i] = fmaf(w[4], b.x, acc[i]);
        acc[i] = fmaf(w[5], b.y, acc[i]);
        acc[i] = fmaf(w[6], b.z, acc[i]);
        acc[i] = fmaf(w[7], b.w, acc[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    if (i < M) {
      float v = acc[i];
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) scores[(size_t)i * C + c] = v;
    }
  }
}

// ------------------------------------------------------------------------------- host side

// Persistent CTAs of the dense head (one per SM, at most one per vocabulary tile).
static int umma_grid(int V) {
  const int sms = sm_count();
  const int tiles = (V + BM - 1) / BM;
  if (sms <= 0) return 0;
  return tiles < sms ? tiles : sms;
}

template <int N>
static sd_status launch_umma(const void *h, const void *w, int M, int d, int V, float *logits,
                             int ld, cudaStream_t st) {
  using C = UCfg<N>;
  static bool attr_set[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(lm_head_umma_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)C::SMEM) != cudaSuccess)
      return SD_ERR_CUDA;
    attr_set[dev] = true;
  }
  CUtensorMap wm, hm;
  if (!encode_tmap_2d_bf16(&wm, w, d, V, (uint64_t)d * 2, BK, BM) ||
      !encode_tmap_2d_bf16(&hm, h, d, M, (uint64_t)d * 2, BK, N))
    return SD_ERR_CUDA;
  Params p{};
  p.M = M;
  p.d = d;
  p.V = V;
  p.ld = ld;
  p.num_tiles = (V + BM - 1) / BM;
  p.kblocks = d / BK;
  p.logits = logits;
  p.status = device_status_word();
  const int grid = umma_grid(V);
  if (grid <= 0) return SD_ERR_CUDA;
  return cuda_status(
      launch(lm_head_umma_kernel<N>, dim3(grid), dim3(C::THREADS), C::SMEM, st, wm, hm, p));
}

// Dense bf16 projection of up to 256 rows.
static sd_status dense_bf16(const void *h, const void *w, int M, int d, int V, float *logits,
                            int ld, cudaStream_t st) {
  if (M <= 16) return launch_umma<16>(h, w, M, d, V, logits, ld, st);
  if (M <= 32) return launch_umma<32>(h, w, M, d, V, logits, ld, st);
  if (M <= 48) return launch_umma<48>(h, w, M, d, V, logits, ld, st);
  if (M <= 64) return launch_umma<64>(h, w, M, d, V, logits, ld, st);
  if (M <= 96) return launch_umma<96>(h, w, M, d, V, logits, ld, st);
  if (M <= 128) return launch_umma<128>(h, w, M, d, V, logits, ld, st);
  if (M <= 192) return launch_umma<192>(h, w, M, d, V, logits, ld, st);
  return launch_umma<256>(h, w, M, d, V, logits, ld, st);
}

static sd_status validate(const sd_head_desc *d) {
  if (!d) return SD_ERR_INVALID_ARG;
  if (d->m < 1 || d->d < 1 || d->vocab < 1) return SD_ERR_INVALID_ARG;
  const int ld = d->ld_logits ? d->ld_logits : d->vocab;
  if (ld < d->vocab) return SD_ERR_INVALID_ARG;
  if (d->dtype != SD_BF16 && d->dtype != SD_F32) return SD_ERR_INVALID_ARG;
  if (d->top_c < 0) return SD_ERR_INVALID_ARG;
  if (d->top_c > 0) {
    if (d->dtype != SD_BF16) return SD_ERR_UNSUPPORTED;
    if (d->n_clusters < 1 || d->cluster_size < 1 ||
        (long long)d->n_clusters * d->cluster_size != d->vocab || d->top_c > d->n_clusters)
      return SD_ERR_INVALID_ARG;
    if (d->top_c > 64 || d->n_clusters > 8192 || d->d > 4096) return SD_ERR_UNSUPPORTED;
  }
  if (d->dtype == SD_BF16 && d->d % 64) return SD_ERR_UNSUPPORTED;
  if (d->dtype == SD_BF16 && (long long)d->vocab >= (1ll << 31)) return SD_ERR_UNSUPPORTED;
  return SD_OK;
}

static size_t ws_size(const sd_head_desc *d) {
  if (validate(d) != SD_OK) return 0;
  if (d->top_c == 0) return 0;
  return round_up((size_t)d->m * d->n_clusters * 4, 256);
}

}  // namespace head
}  // namespace sdv

extern "C" {

size_t sd_lm_head_workspace_size(const sd_head_desc *desc) { return sdv::head::ws_size(desc); }

sd_status sd_lm_head(const sd_head_desc *desc, const void *h, const void *w,
                     const void *centroids, const int32_t *cluster_tokens, float *logits,
                     int32_t *sel_clusters, void *ws, size_t ws_bytes, sd_stream stream) {
  using namespace sdv;
  using namespace sdv::head;
  sd_status s = validate(desc);
  if (s != SD_OK) return s;
  if (!h || !w || !logits) return SD_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const int ld = desc->ld_logits ? desc->ld_logits : desc->vocab;
  if (desc->dtype == SD_F32) {
    Params p{};
    p.M = desc->m;
    p.d = desc->d;
    p.V = desc->vocab;
    p.ld = ld;
    p.logits = logits;
    return cuda_status(launch(lm_head_f32_kernel, dim3((desc->vocab + 7) / 8), dim3(256), 0, st,
                              (const float *)h, (const float *)w, p));
  }
  if (!aligned16(h) || !aligned16(w)) return SD_ERR_INVALID_ARG;
  const size_t hrow = (size_t)desc->d * 2;
  if (desc->top_c == 0) {
    for (int m0 = 0; m0 < desc->m; m0 += 256) {
      const int mm = desc->m - m0 < 256 ? desc->m - m0 : 256;
      s = dense_bf16((const uint8_t *)h + m0 * hrow, w, mm, desc->d, desc->vocab,
                     logits + (size_t)m0 * ld, ld, st);
      if (s != SD_OK) return s;
    }
    return SD_OK;
  }
  // clustered
  if (!centroids || !cluster_tokens || !sel_clusters || !aligned16(centroids))
    return SD_ERR_INVALID_ARG;
  if (!ws || ws_bytes < ws_size(desc)) return SD_ERR_WORKSPACE;
  float *scores = reinterpret_cast<float *>(ws);
  const int C = desc->n_clusters;
  if (desc->m <= 16 && desc->d <= 1024 && (size_t)desc->m * desc->d * 4 <= 48 * 1024) {
    if (launch(centroid_scores_kernel, dim3((C + 7) / 8), dim3(256),
               (size_t)desc->m * desc->d * 4, st, (const __nv_bfloat16 *)h,
               (const __nv_bfloat16 *)centroids, desc->m, desc->d, C, scores) != cudaSuccess)
      return SD_ERR_CUDA;
  } else {
    for (int m0 = 0; m0 < desc->m; m0 += 256) {
      const int mm = desc->m - m0 < 256 ? desc->m - m0 : 256;
      s = dense_bf16((const uint8_t *)h + m0 * hrow, centroids, mm, desc->d, C,
                     scores + (size_t)m0 * C, C, st);
      if (s != SD_OK) return s;
    }
  }
  // selection (block 0 of each row) and the -inf fill of the row (the other blocks): about
  // one wave of blocks over all rows
  const int vec4 = aligned16(logits) && desc->vocab % 4 == 0 && ld % 4 == 0;
  const int per_row = (desc->vocab / (vec4 ? 4 : 1) + kSelThreads - 1) / kSelThreads;
  const int sms = sm_count();
  int fill_blocks = ((sms > 0 ? sms : 148) + desc->m - 1) / desc->m;
  if (fill_blocks > per_row) fill_blocks = per_row;
  if (fill_blocks < 1) fill_blocks = 1;
  const size_t sel_smem = (size_t)C * 4;
  if (sel_smem > 48 * 1024 &&
      cudaFuncSetAttribute(select_fill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)sel_smem) != cudaSuccess)
    return SD_ERR_CUDA;
  if (launch(select_fill_kernel, dim3(1 + fill_blocks, desc->m), dim3(kSelThreads), sel_smem, st,
             (const float *)scores, C, desc->top_c, sel_clusters, logits, desc->vocab, ld,
             vec4) != cudaSuccess)
    return SD_ERR_CUDA;
  if (desc->d <= 1024 && desc->cluster_size % kClTok == 0 && aligned16(cluster_tokens)) {
    static bool attr_set[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
      if (cudaFuncSetAttribute(cluster_logits_tma_kernel,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kClSmem) != cudaSuccess)
        return SD_ERR_CUDA;
      attr_set[dev] = true;
    }
    return cuda_status(launch(cluster_logits_tma_kernel, dim3(sms > 0 ? sms : 148),
                              dim3(32 * (kClWarps + 1)), kClSmem, st, (const __nv_bfloat16 *)h,
                              (const __nv_bfloat16 *)w, cluster_tokens,
                              (const int32_t *)sel_clusters, desc->m, desc->top_c,
                              desc->cluster_size, desc->d, C, desc->vocab, ld, logits,
                              device_status_word()));
  }
  // persistent warps: as many 8-warp CTAs as fit on the device at once
  int occ = 0;
  if (desc->d <= 1024)
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, cluster_logits_kernel<4, 4>, 256, 0);
  else
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, cluster_logits_kernel<16, 2>, 256, 0);
  const dim3 grid((occ > 0 ? occ : 1) * (sms > 0 ? sms : 148));
  if (desc->d <= 1024)
    s = cuda_status(launch(cluster_logits_kernel<4, 4>, grid, dim3(256), 0, st,
                           (const __nv_bfloat16 *)h, (const __nv_bfloat16 *)w, cluster_tokens,
                           (const int32_t *)sel_clusters, desc->m, desc->top_c,
                           desc->cluster_size, desc->d, C, desc->vocab, ld, logits,
                           device_status_word()));
  else
    s = cuda_status(launch(cluster_logits_kernel<16, 2>, grid, dim3(256), 0, st,
                           (const __nv_bfloat16 *)h, (const __nv_bfloat16 *)w, cluster_tokens,
                           (const int32_t *)sel_clusters, desc->m, desc->top_c,
                           desc->cluster_size, desc->d, C, desc->vocab, ld, logits,
                           device_status_word()));
  return s;
}

}  // extern "C"
