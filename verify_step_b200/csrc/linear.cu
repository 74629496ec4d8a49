// Dense layers of the drafter and of the target: one projection of a few token rows against a
// bf16 weight matrix, with an RMSNorm / embedding-gather prologue and a store, residual-add or
// gated-GELU epilogue (sm_100a).
//
// "Gemma 4 MTP: drafter drafts, target verifies", section "drafter internal architecture": the
// drafter runs 4 transformer layers on the target's last-layer activation and its own token
// embedding, and the target runs its layers over the k+1 verified positions.  With B = 8 token
// rows a projection is a matrix-vector product in all but name:
// 8 FLOPs per weight byte, so the weights' single pass through HBM bounds it.  The kernel
// streams each CTA's W rows into shared memory with a few large TMA tensor copies (completing on
// mbarriers), feeds mma.sync from there and keeps the few token rows in
// shared memory in fragment order; the K dimension is split over the CTAs of a thread-block
// cluster and reduced through distributed shared memory, so the result needs no workspace and
// does not depend on the launch.
//
// Fragment trick: a thread's 16-byte read holds 8 consecutive columns 8q .. 8q+7 of one W row.
// The two m16n8k16 steps of a 32-column chunk take columns {8q..8q+3} and {8q+4..8q+7} as their
// logical k indices {2q, 2q+1, 2q+8, 2q+9}; the token rows are staged with the same column
// mapping, so each product pairs the same physical column on both sides.
#include <algorithm>

#include "common.cuh"
#include "host.cuh"

namespace sdv {
namespace lin {

constexpr int kWarpsN = 2;                 // warps along W rows (16 rows each)
constexpr int kWarpsK = 4;                 // warps along K inside a CTA
constexpr int kThreads = 32 * kWarpsN * kWarpsK;
constexpr int kRows = 16 * kWarpsN;        // W rows per CTA
constexpr int kMaxM = 64;

struct Params {
  int m, n, k, k_x, x_f32;
  long long ld_x;
  const void *x;
  const __nv_bfloat16 *W;
  const __nv_bfloat16 *table;
  long long ld_table, table_rows, ld_tokens;
  const int32_t *tokens;
  const int32_t *token_sel;
  const float *gain;
  float eps;
  int epi, out_f32;
  long long ld_out;
  void *out;
  __nv_bfloat16 *norm_out;
  long long ld_norm_out;
  int splits;        // CTAs per cluster, each taking a contiguous share of the k chunks
  int piece;         // chunks staged per piece
  int *status;
};

__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ float gelu_tanh(float z) {
  return 0.5f * z * (1.f + tanhf(0.7978845608028654f * (z + 0.044715f * z * z * z)));
}

__device__ __forceinline__ float4 bf16x4_to_f4(uint2 u) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

// Four consecutive input columns col .. col+3 of row r, before normalisation (zeros for a row
// past m or an invalid token).  Branch-free apart from the loads' own predicates, so that a
// thread's loads in an unrolled loop are all in flight together.
template <bool XF32>
__device__ __forceinline__ float4 input4(const Params &p, int r, int col, int tok) {
  const bool in_x = r < p.m && col < p.k_x;
  const bool in_t = r < p.m && col >= p.k_x && tok >= 0;
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (XF32) {
    if (in_x)
      v = *reinterpret_cast<const float4 *>(static_cast<const float *>(p.x) + r * p.ld_x + col);
  } else if (in_x) {
    v = bf16x4_to_f4(*reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(p.x) +
                                                      r * p.ld_x + col));
  }
  if (in_t) v = bf16x4_to_f4(*reinterpret_cast<const uint2 *>(p.table + tok * p.ld_table +
                                                              (col - p.k_x)));
  return v;
}

constexpr int kLd = 8;  // input loads in flight per thread in the prologue

constexpr int kGroup = 8;     // chunks per tensor-copy group (one mbarrier each)
constexpr int kMaxPiece = 32; // chunks staged per piece
constexpr int kMaxGroups = kMaxPiece / kGroup;
constexpr int kGroupBytes = kRows * kGroup * 64;  // 16 KB of weights per group

// Shared-memory plan of a CTA for a piece of P chunks: the weights (one 16 KB region per group
// of 8 chunks), the token rows in fragment order, then the partial sums; the reduction buffer
// reuses the first two regions.
__host__ __device__ constexpr int w_bytes(int P) { return (P + kGroup - 1) / kGroup * kGroupBytes; }
__host__ __device__ constexpr int region_a(int P, int NT) {
  return w_bytes(P) + NT * P * 512 > kWarpsK * kRows * NT * 32 ? w_bytes(P) + NT * P * 512
                                                               : kWarpsK * kRows * NT * 32;
}

// grid: (ceil(n / 32) row blocks) x splits CTAs, clusters of `splits` along x; NT token groups
// of 8 (m <= 8 NT).  One thread brings the CTA's weight rows into shared memory with TMA tensor
// copies (no multicast): a full group of 8 chunks is one [32 rows x 256 columns] box (row-major,
// 512 bytes a row), a partial group one [32 x 32] box per chunk (64 bytes a row); each group
// completes on its own mbarrier.  Every warp then takes a 16-row half of the rows and a quarter
// of the chunks.  Rows past n arrive as zeros (tensor out-of-bounds fill).
template <int NT, bool XF32>
__global__ void __launch_bounds__(kThreads, NT <= 2 ? 2 : 1)
    linear_kernel(const __grid_constant__ CUtensorMap wmap_big,
                  const __grid_constant__ CUtensorMap wmap_small, const Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_inv[kMaxM];
  __shared__ int s_tok[kMaxM];
  __shared__ __align__(8) uint64_t s_bar[kMaxGroups];
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wr = warp % kWarpsN, wk = warp / kWarpsN;
  const int g = lane >> 2, q = lane & 3;
  const int S = p.splits;
  const int rank = S > 1 ? (int)cluster_ctarank() : 0;
  const int rb = blockIdx.x / S;
  const int row0 = rb * kRows;
  const int box_rows = min(kRows, p.n);  // rows of every tensor box (the map's box height)
  const int C = p.k >> 5;
  const int c_begin = (int)((long long)C * rank / S);
  const int c_end = (int)((long long)C * (rank + 1) / S);
  const int P = p.piece;
  uint8_t *wsm = smem;
  uint2 *xs = reinterpret_cast<uint2 *>(smem + w_bytes(P));
  float *part = reinterpret_cast<float *>(smem + region_a(P, NT));

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxGroups; ++i) mbar_init(&s_bar[i], 1);
    fence_mbar_init();
  }
  __syncthreads();

  // thread 0: tensor copies of the weight rows of chunks pc0 .. pc0+np-1
  auto issue = [&](int pc0, int np) {
    if (threadIdx.x != 0) return;
    const int groups = (np + kGroup - 1) / kGroup;
    for (int gi = 0; gi < groups; ++gi) {
      const int cnt = min(kGroup, np - gi * kGroup);
      const int col = (pc0 + gi * kGroup) * 32;
      mbar_arrive_expect_tx(&s_bar[gi], (uint32_t)(box_rows * cnt * 64));
      if (cnt == kGroup) {
        tma_load_2d(wsm + gi * kGroupBytes, &wmap_big, &s_bar[gi], col, row0);
      } else {
        for (int c = 0; c < cnt; ++c)
          tma_load_2d(wsm + gi * kGroupBytes + c * (kRows * 64), &wmap_small, &s_bar[gi],
                      col + c * 32, row0);
      }
    }
  };
  // the weights are requested before anything else: the prologue below (token ids, row
  // statistics, staging of the token rows) runs under their HBM latency
  issue(c_begin, min(P, c_end - c_begin));

  // ---- token ids and row statistics
  if (threadIdx.x < p.m) {
    const int r = threadIdx.x;
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
    s_tok[threadIdx.x] = t;
  }
  __syncthreads();
  if (p.gain != nullptr) {
    for (int r = warp; r < p.m; r += kThreads / 32) {
      const int tok = s_tok[r];
      float ss = 0.f;
      for (int c0 = lane * 4; c0 < p.k; c0 += 128 * kLd) {
        float4 v[kLd];
#pragma unroll
        for (int u = 0; u < kLd; ++u)
          v[u] = c0 + 128 * u < p.k ? input4<XF32>(p, r, c0 + 128 * u, tok)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < kLd; ++u)
          ss += v[u].x * v[u].x + v[u].y * v[u].y + v[u].z * v[u].z + v[u].w * v[u].w;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) s_inv[r] = rsqrtf(ss / (float)p.k + p.eps);
    }
  }

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  const bool active = row0 + wr * 16 < p.n;
  uint32_t parity = 0;
  bool timed_out = false;

  for (int pc0 = c_begin; pc0 < c_end; pc0 += P) {
    const int np = min(P, c_end - pc0);
    if (pc0 != c_begin) {
      __syncthreads();  // every warp is done with the previous piece's rows and fragments
      issue(pc0, np);
    }
    __syncthreads();  // s_inv ready
    // ---- stage the token rows of chunks pc0 .. pc0+np-1 in fragment order
    const int total = NT * np * 64;
    for (int base = threadIdx.x; base < total; base += kThreads * kLd) {
      float4 v[kLd];
#pragma unroll
      for (int u = 0; u < kLd; ++u) {
        const int idx = base + kThreads * u;
        const int ln = idx & 31, s = (idx >> 5) & 1, rest = idx >> 6;
        const int cc = rest % np, tg = rest / np;
        const int r = idx < total ? tg * 8 + (ln >> 2) : p.m;  // rows past m read nothing
        const int col = (pc0 + cc) * 32 + (ln & 3) * 8 + s * 4;
        v[u] = input4<XF32>(p, r, col, r < p.m ? s_tok[r] : -1);
      }
#pragma unroll
      for (int u = 0; u < kLd; ++u) {
        const int idx = base + kThreads * u;
        if (idx >= total) break;
        const int ln = idx & 31, s = (idx >> 5) & 1, rest = idx >> 6;
        const int cc = rest % np, tg = rest / np;
        const int r = tg * 8 + (ln >> 2);
        const int col = (pc0 + cc) * 32 + (ln & 3) * 8 + s * 4;
        uint2 v2 = make_uint2(0u, 0u);
        if (r < p.m) {
          float4 x4 = v[u];
          if (p.gain != nullptr) {
            const float inv = s_inv[r];
            const float4 gg = *reinterpret_cast<const float4 *>(p.gain + col);
            x4 = make_float4(x4.x * inv * gg.x, x4.y * inv * gg.y, x4.z * inv * gg.z,
                             x4.w * inv * gg.w);
          }
          v2 = make_uint2(pack_bf16x2(x4.x, x4.y), pack_bf16x2(x4.z, x4.w));
          if (p.norm_out != nullptr && rb == 0)
            *reinterpret_cast<uint2 *>(p.norm_out + r * p.ld_norm_out + col) = v2;
        }
        xs[((tg * P + cc) * 2 + s) * 32 + ln] = v2;
      }
    }
    __syncthreads();
    // ---- products: chunk cc of the piece is in group cc / 8
    const int row = wr * 16 + g;
    const int groups = (np + kGroup - 1) / kGroup;
    for (int gi = 0; gi < groups; ++gi) {
      if (!mbar_wait_timed(&s_bar[gi], parity)) timed_out = true;
      const bool full = np - gi * kGroup >= kGroup;
      const uint8_t *gbase = wsm + gi * kGroupBytes;
#pragma unroll
      for (int u = 0; u < kGroup / kWarpsK; ++u) {
        const int c8 = wk + kWarpsK * u;
        const int cc = gi * kGroup + c8;
        if (active && cc < np) {
          // [32 x 256] box: row r at r * 512; [32 x 32] box of chunk c8 at c8 * 2048, row r at
          // r * 64
          const uint8_t *w_lo = full ? gbase + row * 512 + c8 * 64 + q * 16
                                     : gbase + c8 * (kRows * 64) + row * 64 + q * 16;
          const int hi_off = full ? 8 * 512 : 8 * 64;
          const uint4 lo = *reinterpret_cast<const uint4 *>(w_lo);
          const uint4 hi = *reinterpret_cast<const uint4 *>(w_lo + hi_off);
          const uint32_t f0[4] = {lo.x, hi.x, lo.y, hi.y};
          const uint32_t f1[4] = {lo.z, hi.z, lo.w, hi.w};
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const uint2 b_0 = xs[((t * P + cc) * 2 + 0) * 32 + lane];
            const uint2 b_1 = xs[((t * P + cc) * 2 + 1) * 32 + lane];
            mma_bf16_16816(acc[t], f0, b_0.x, b_0.y);
            mma_bf16_16816(acc[t], f1, b_1.x, b_1.y);
          }
        }
      }
    }
    parity ^= 1u;
  }
  if (timed_out) record_status(p.status, SD_ERR_TIMEOUT);

  // ---- reduce the kWarpsK partial sums of each warp row in shared memory (fixed order)
  __syncthreads();
  float *red = reinterpret_cast<float *>(smem);  // [kWarpsK][kRows][NT * 8]
  constexpr int MT8 = NT * 8;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    float *base = red + ((size_t)wk * kRows + wr * 16) * MT8 + t * 8 + 2 * q;
    base[g * MT8] = acc[t][0];
    base[g * MT8 + 1] = acc[t][1];
    base[(g + 8) * MT8] = acc[t][2];
    base[(g + 8) * MT8 + 1] = acc[t][3];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kRows * MT8; i += kThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarpsK; ++w) v += red[(size_t)w * kRows * MT8 + i];
    part[i] = v;
  }
  if (S > 1)
    cluster_sync();  // every CTA's partial is complete and visible to the cluster
  else
    __syncthreads();

  // ---- sum over the cluster in rank order and apply the epilogue; CTA `rank` takes a
  // contiguous share of the output units (rows, or gated features)
  const int units = p.epi == SD_EPI_GEGLU ? kRows / 2 : kRows;
  const int u0 = units * rank / S, u1 = units * (rank + 1) / S;
  const int nu = u1 - u0;
  const uint32_t part_s = smem_u32(part);
  // sum of element idx of the partials over the cluster's CTAs, in rank order (the DSMEM loads
  // are all issued before the first add; ranks past S add an exact zero)
  auto cluster_sum = [&](int idx) -> float {
    if (S == 1) return part[idx];
    float v[8];
#pragma unroll
    for (int c = 0; c < 8; ++c)
      v[c] = c < S ? ld_dsmem_f32(dsmem_addr(part_s + (uint32_t)idx * 4u, c)) : 0.f;
    float y = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) y += v[c];
    return y;
  };
  for (int i = threadIdx.x; i < nu * p.m; i += kThreads) {
    const int tok = i / nu, unit = u0 + i % nu;
    if (p.epi == SD_EPI_GEGLU) {
      const int f = rb * (kRows / 2) + unit;
      if (f >= p.n / 2) continue;
      const int rg = (unit >> 3) * 16 + (unit & 7), ru = rg + 8;
      const float yg = cluster_sum(rg * MT8 + tok);
      const float yu = cluster_sum(ru * MT8 + tok);
      static_cast<__nv_bfloat16 *>(p.out)[tok * p.ld_out + f] =
          __float2bfloat16_rn(gelu_tanh(yg) * yu);
    } else {
      const int row = row0 + unit;
      if (row >= p.n) continue;
      const float y = cluster_sum(unit * MT8 + tok);
      const long long o = tok * p.ld_out + row;
      if (p.epi == SD_EPI_ADD)
        static_cast<float *>(p.out)[o] += y;
      else if (p.out_f32)
        static_cast<float *>(p.out)[o] = y;
      else
        static_cast<__nv_bfloat16 *>(p.out)[o] = __float2bfloat16_rn(y);
    }
  }
  if (S > 1) cluster_sync();  // no CTA leaves while another still reads its partial
}

template <int NT, bool XF32>
struct Launcher {
  static size_t smem_bytes(int piece) {
    return (size_t)region_a(piece, NT) + (size_t)kRows * NT * 8 * 4;
  }
  static sd_status launch(const CUtensorMap &big, const CUtensorMap &small, const Params &p,
                          int row_blocks, cudaStream_t st) {
    const size_t smem = smem_bytes(p.piece);
    static int configured[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || configured[dev] != dev + 1) {
      if (cudaFuncSetAttribute(linear_kernel<NT, XF32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem_bytes(kMaxPiece)) != cudaSuccess)
        return SD_ERR_CUDA;
      if (dev < 64) configured[dev] = dev + 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(row_blocks * p.splits);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute a[2];
    int na = 0;
    if (p.splits > 1) {
      a[na].id = cudaLaunchAttributeClusterDimension;
      a[na].val.clusterDim.x = p.splits;
      a[na].val.clusterDim.y = 1;
      a[na].val.clusterDim.z = 1;
      ++na;
    }
    if (pdl_enabled()) {
      a[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      a[na].val.programmaticStreamSerializationAllowed = 1;
      ++na;
    }
    cfg.attrs = a;
    cfg.numAttrs = na;
    return cuda_status(cudaLaunchKernelEx(&cfg, linear_kernel<NT, XF32>, big, small, p));
  }
};

}  // namespace lin
}  // namespace sdv

extern "C" sd_status sd_linear(const sd_linear_desc *d, const void *x, const void *W, void *out,
                               const void *table, const int32_t *tokens,
                               const int32_t *token_sel, sd_stream stream) {
  using namespace sdv;
  using namespace sdv::lin;
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

  Params p{};
  p.m = d->m;
  p.n = d->n;
  p.k = d->k;
  p.k_x = k_x;
  p.x_f32 = d->x_dtype == SD_F32;
  p.ld_x = d->ld_x;
  p.x = x;
  p.W = static_cast<const __nv_bfloat16 *>(W);
  p.table = static_cast<const __nv_bfloat16 *>(table);
  p.ld_table = d->ld_table;
  p.table_rows = d->table_rows;
  p.ld_tokens = d->ld_tokens;
  p.tokens = tokens;
  p.token_sel = token_sel;
  p.gain = d->norm_gain;
  p.eps = d->norm_eps;
  p.epi = d->epilogue;
  p.out_f32 = d->out_dtype == SD_F32;
  p.ld_out = d->ld_out;
  p.out = out;
  p.norm_out = static_cast<__nv_bfloat16 *>(d->norm_out);
  p.ld_norm_out = d->ld_norm_out;
  p.status = device_status_word();

  // Split K over a cluster until the grid covers about two CTAs per SM.
  const int row_blocks = (d->n + kRows - 1) / kRows;
  const int chunks = d->k / 32;
  const int target = 2 * std::max(sm_count(), 1);
  int S = 1;
  while (S < 8 && row_blocks * S * 2 <= target + target / 4 && chunks >= 8 * S) S *= 2;
  p.splits = S;
  const int NT = d->m <= 8 ? 1 : d->m <= 16 ? 2 : d->m <= 32 ? 4 : 8;
  const int per_cta = (chunks + S - 1) / S;
  p.piece = std::max(1, std::min(per_cta, kMaxPiece));
  // weight boxes: [32 rows x 256 columns] for a full group of 8 chunks, [32 x 32] for one chunk
  CUtensorMap big, small;
  const uint32_t box_rows = (uint32_t)std::min(kRows, d->n);
  if (!encode_tmap_2d_bf16(&big, W, (uint64_t)d->k, (uint64_t)d->n, (uint64_t)d->k * 2,
                           (uint32_t)std::min(kGroup * 32, d->k), box_rows, false) ||
      !encode_tmap_2d_bf16(&small, W, (uint64_t)d->k, (uint64_t)d->n, (uint64_t)d->k * 2, 32,
                           box_rows, false))
    return SD_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  if (p.x_f32) {
    switch (NT) {
      case 1: return Launcher<1, true>::launch(big, small, p, row_blocks, st);
      case 2: return Launcher<2, true>::launch(big, small, p, row_blocks, st);
      case 4: return Launcher<4, true>::launch(big, small, p, row_blocks, st);
      default: return Launcher<8, true>::launch(big, small, p, row_blocks, st);
    }
  }
  switch (NT) {
    case 1: return Launcher<1, false>::launch(big, small, p, row_blocks, st);
    case 2: return Launcher<2, false>::launch(big, small, p, row_blocks, st);
    case 4: return Launcher<4, false>::launch(big, small, p, row_blocks, st);
    default: return Launcher<8, false>::launch(big, small, p, row_blocks, st);
  }
}
