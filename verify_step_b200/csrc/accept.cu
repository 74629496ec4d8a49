// Lossless acceptance of k drafts, correction / bonus draw, greedy rule (sm_100a).
//
// The rule (pages cite Leviathan et al. for it: Google blog translation, section "how
// speculative decoding works"; property stated in "Gemma 4 MTP: drafter drafts, target
// verifies", section "basic structure of speculative decoding"): accept d_i iff
// u_i < p_i(d_i) / q_i(d_i); at the first rejection emit x ~ norm(max(0, p_i - q_i)); if all
// are accepted emit the bonus x ~ p_{k+1}.  T = 0: accept iff d_i == argmax, emit argmax.
//
// Two kernels, both bandwidth-bound scans of float32 logits (vectorised 16-byte loads):
//  1. accept_stats: one CTA per (row, 8192-token chunk): online max / sum of exp(x / T)
//     (T > 0) or the top two values and the argmax (T = 0) of the chunk.
//  2. accept_draw: one CTA per (sequence, chunk).  Every CTA merges the row statistics in
//     chunk order, takes the acceptance decisions (a handful of single-element reads and
//     Philox uniforms), then runs the exponential race of the draw row over its chunk:
//     key_v = ln w_v - ln(-ln(1 - V_v)), V_v the token's Philox uniform, for both the
//     residual weights max(0, p - q) and for p (the fallback when the residual is empty).
//     The last CTA of a sequence (atomic ticket; no waiting) merges the chunk winners in chunk
//     order, lowest token id first on ties, and writes the outputs.
#include <cfloat>
#include <mutex>

#include "common.cuh"
#include "host.cuh"
#include "philox.cuh"

namespace sdv {
namespace acc {

constexpr int kChunk = 8192;      // tokens per CTA of the statistics pass
constexpr int kDrawSlots = 592;  // draw CTAs aimed at: one wave at 4 CTAs on each of 148 SMs
constexpr int kThreads = 256;
constexpr float kMargin = 1e-4f;

struct Params {
  int B, k, V, n_q, ld_t, ld_d, ld_o, purpose, nchunks, stats_chunk, ndraw, draw_chunk, rows_t,
      rows_total;
  float T;
  unsigned long long seed;
  unsigned long long step;
  const unsigned long long *step_ptr;  // nullable: step = *step_ptr + step
  const float *z;
  const float *y;
  const int32_t *drafts;
  int32_t *n_acc;
  int32_t *out;
  int32_t *margin;
  float4 *stats;   // [rows_total][nchunks]
  int stats_row0, stats_rows;  // rows the statistics pass computes
  // optional producer partials (max, sum exp) per slot: target rows, draft rows
  const float2 *tstats;
  int tslots, tld;
  const float2 *dstats;
  int dslots, dld;
  float2 *sout;  // plain draws: partials of the drawn row per draw chunk
  int sld;
  float4 *cand;    // [B][ndraw][2]
  unsigned int *counters;  // [B]
  int *status;
};

// E = -ln(1 - V) for V in [0, 1): the series V + V^2/2 + ... + V^8/8 below 1/16 (truncation
// below 3e-11 relative), else -ln(1 - V) with 1 - V formed exactly or within 2^-25 and the fast
// logarithm (absolute error below 4e-7, i.e. below 6e-6 relative to E >= 0.0645).
__device__ __forceinline__ float neg_log1m(float V) {
  if (V < 0.0625f) {
    float t = 0.125f;
    t = fmaf(V, t, 0.14285714f);
    t = fmaf(V, t, 0.16666667f);
    t = fmaf(V, t, 0.2f);
    t = fmaf(V, t, 0.25f);
    t = fmaf(V, t, 0.33333333f);
    t = fmaf(V, t, 0.5f);
    t = fmaf(V, t, 1.f);
    return V * t;
  }
  return -__logf(1.f - V);
}

struct Cand {  // best and runner-up key of a race, best token id
  float g1, g2;
  int v1;
};

__device__ __forceinline__ void cand_push(Cand &c, float g, int v) {
  // tokens arrive in increasing v per thread; strict > keeps the lowest id on ties
  if (g > c.g1) {
    c.g2 = c.g1;
    c.g1 = g;
    c.v1 = v;
  } else if (g > c.g2) {
    c.g2 = g;
  }
}

__device__ __forceinline__ Cand cand_merge(const Cand &a, const Cand &b) {
  // a holds lower token ids than b when ids tie in key
  Cand r;
  if (b.g1 > a.g1 || (b.g1 == a.g1 && b.v1 < a.v1 && b.v1 >= 0)) {
    r.g1 = b.g1;
    r.v1 = b.v1;
    r.g2 = fmaxf(b.g2, a.g1);
  } else {
    r.g1 = a.g1;
    r.v1 = a.v1;
    r.g2 = fmaxf(a.g2, b.g1);
  }
  return r;
}

__device__ __forceinline__ Cand cand_shfl(const Cand &c, int off) {
  Cand o;
  o.g1 = __shfl_xor_sync(0xffffffffu, c.g1, off);
  o.g2 = __shfl_xor_sync(0xffffffffu, c.g2, off);
  o.v1 = __shfl_xor_sync(0xffffffffu, c.v1, off);
  return o;
}

// (max, sum exp(x - max)) pairs
__device__ __forceinline__ void ms_merge(float &m, float &s, float m2, float s2) {
  const float mm = fmaxf(m, m2);
  if (mm == -INFINITY) return;
  s = s * expf(m - mm) + s2 * expf(m2 - mm);
  m = mm;
}

__device__ __forceinline__ const float *row_ptr(const Params &p, int r) {
  return r < p.rows_t ? p.z + (size_t)r * p.ld_t : p.y + (size_t)(r - p.rows_t) * p.ld_d;
}

__global__ void __launch_bounds__(kThreads) accept_stats_kernel(const Params p) {
  pdl_wait();  // many waves: no early trigger, so the next kernel does not take their slots
  const int r = p.stats_row0 + blockIdx.x, c = blockIdx.y;
  if (c == 0 && blockIdx.x == 0)
    for (int b = threadIdx.x; b < p.B; b += blockDim.x) p.counters[b] = 0u;
  const float *row = row_ptr(p, r);
  const int v0 = c * p.stats_chunk;
  const int v1 = min(p.V, v0 + p.stats_chunk);
  const float4 *row4 = reinterpret_cast<const float4 *>(row + v0);
  const int n4 = (v1 - v0) >> 2;
  __shared__ float4 red[kThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (p.T > 0.f) {
    // kChunk tokens at a time: all of this thread's values first (independent loads), then
    // their max, then the sum, merged online across batches
    constexpr int PER = kChunk / 4 / kThreads;
    float m = -INFINITY, s = 0.f;
    for (int base = 0; base < n4; base += PER * kThreads) {
      float4 x[PER];
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        const int i = base + threadIdx.x + u * kThreads;
        x[u] = i < n4 ? __ldg(row4 + i)
                      : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      }
      if (p.T != 1.f) {
#pragma unroll
        for (int u = 0; u < PER; ++u)
          x[u] = make_float4(x[u].x / p.T, x[u].y / p.T, x[u].z / p.T, x[u].w / p.T);
      }
      float mb = -INFINITY, sb = 0.f;
#pragma unroll
      for (int u = 0; u < PER; ++u)
        mb = fmaxf(mb, fmaxf(fmaxf(x[u].x, x[u].y), fmaxf(x[u].z, x[u].w)));
      if (mb != -INFINITY) {
        constexpr float L2E = 1.4426950408889634f;
#pragma unroll
        for (int u = 0; u < PER; ++u)
          sb += (exp2f((x[u].x - mb) * L2E) + exp2f((x[u].y - mb) * L2E)) +
                (exp2f((x[u].z - mb) * L2E) + exp2f((x[u].w - mb) * L2E));
      }
      ms_merge(m, s, mb, sb);
    }
    for (int off = 16; off > 0; off >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
      const float s2 = __shfl_xor_sync(0xffffffffu, s, off);
      ms_merge(m, s, m2, s2);
    }
    if (lane == 0) red[warp] = make_float4(m, s, 0.f, 0.f);
    __syncthreads();
    if (threadIdx.x == 0) {
      float M = red[0].x, S = red[0].y;
      for (int w = 1; w < kThreads / 32; ++w) ms_merge(M, S, red[w].x, red[w].y);
      p.stats[(size_t)r * p.nchunks + c] = make_float4(M, S, 0.f, 0.f);
    }
  } else {
    Cand cd{-INFINITY, -INFINITY, -1};
    for (int i = threadIdx.x; i < n4; i += kThreads) {
      const float4 x4 = __ldg(row4 + i);
      const int v = v0 + 4 * i;
      cand_push(cd, x4.x, v);
      cand_push(cd, x4.y, v + 1);
      cand_push(cd, x4.z, v + 2);
      cand_push(cd, x4.w, v + 3);
    }
    for (int off = 16; off > 0; off >>= 1) {
      const Cand o = cand_shfl(cd, off);
      // lane order is not token order inside a warp: break ties by id explicitly
      cd = (lane & off) ? cand_merge(o, cd) : cand_merge(cd, o);
    }
    if (lane == 0) red[warp] = make_float4(cd.g1, __int_as_float(cd.v1), cd.g2, 0.f);
    __syncthreads();
    if (threadIdx.x == 0) {
      Cand t{red[0].x, red[0].z, __float_as_int(red[0].y)};
      for (int w = 1; w < kThreads / 32; ++w) {
        Cand o{red[w].x, red[w].z, __float_as_int(red[w].y)};
        t = cand_merge(t, o);
      }
      p.stats[(size_t)r * p.nchunks + c] = make_float4(t.g1, __int_as_float(t.v1), t.g2, 0.f);
    }
  }
}

// Merged statistics of one row, computed by a full warp (every lane gets the result):
// (max, sum) for T > 0; (top1, argmax, top2) for T = 0.  The argmax merge breaks ties by the
// lower token id, so it does not depend on the merge order.
__device__ __forceinline__ float4 row_stats_warp(const Params &p, int r) {
  const int lane = threadIdx.x & 31;
  const float4 *st = p.stats + (size_t)r * p.nchunks;
  if (p.T > 0.f) {
    float M = -INFINITY, S = 0.f;
    const bool target = r < p.rows_t;
    const float2 *ext = target ? p.tstats : p.dstats;
    if (ext != nullptr) {  // partials from the rows' producers
      const int slots = target ? p.tslots : p.dslots;
      const float2 *e = ext + (size_t)(target ? r : r - p.rows_t) * (target ? p.tld : p.dld);
      for (int c = lane; c < slots; c += 32) {
        const float2 v = e[c];
        ms_merge(M, S, v.x, v.y);
      }
    } else {
      for (int c = lane; c < p.nchunks; c += 32) ms_merge(M, S, st[c].x, st[c].y);
    }
    for (int off = 16; off > 0; off >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, M, off);
      const float s2 = __shfl_xor_sync(0xffffffffu, S, off);
      ms_merge(M, S, m2, s2);
    }
    return make_float4(M, S, 0.f, 0.f);
  }
  Cand t{-INFINITY, -INFINITY, -1};
  for (int c = lane; c < p.nchunks; c += 32)
    t = cand_merge(t, Cand{st[c].x, st[c].z, __float_as_int(st[c].y)});
  for (int off = 16; off > 0; off >>= 1) t = cand_merge(t, cand_shfl(t, off));
  return make_float4(t.g1, __int_as_float(t.v1), t.g2, 0.f);
}

__global__ void __launch_bounds__(kThreads) accept_draw_kernel(const Params p) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x, c = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __shared__ int s_a, s_flag;
  __shared__ float s_mz, s_isz, s_my, s_isy;
  __shared__ float4 red[2][kThreads / 32];
  __shared__ float2 s_part[kThreads / 32];  // plain draws: per-warp softmax partials
  __shared__ int s_last;
  __shared__ uint32_t s_step;
  __shared__ float s_top1, s_top2;
  __shared__ int s_arg;
  __shared__ float4 s_rows[32];  // merged statistics: target rows 0..k, then draft rows 0..k-1

  // ---- statistics of every row this sequence may need, one warp per row (in parallel).  A
  // plain draw (k = 0, T > 0) needs none: the race keys of p are unnormalised logits.
  const int n_rows = (p.k == 0 && p.T > 0.f) ? 0 : p.n_q + (p.T > 0.f ? p.k : 0);
  for (int ri = warp; ri < n_rows; ri += kThreads / 32) {
    const int r = ri < p.n_q ? b * p.n_q + ri : p.rows_t + b * p.k + (ri - p.n_q);
    const float4 st = row_stats_warp(p, r);
    if (lane == 0) s_rows[ri] = st;
  }
  if (threadIdx.x == 0) s_step = (uint32_t)(p.step + (p.step_ptr != nullptr ? *p.step_ptr : 0ull));
  __syncthreads();

  // ---- acceptance tests of the k drafts in parallel (lane i-1 tests draft i), first rejection
  if (threadIdx.x < 32) {
    bool acc = true;
    int flag = 0;
    if (lane < p.k) {
      const int i = lane + 1;
      const int d = p.drafts[(size_t)b * p.k + i - 1];
      const int rt = b * p.n_q + i - 1;
      const float4 sz = s_rows[i - 1];
      if (d < 0 || d >= p.V) {
        record_status(p.status, SD_ERR_DEVICE);
        acc = false;
      } else if (p.T > 0.f) {
        const float4 sy = s_rows[p.n_q + i - 1];
        const float pd = expf(p.z[(size_t)rt * p.ld_t + d] / p.T - sz.x) / sz.y;
        const float qd =
            expf(p.y[((size_t)b * p.k + i - 1) * p.ld_d + d] / p.T - sy.x) / sy.y;
        const float ratio = qd > 0.f ? pd / qd : (pd > 0.f ? INFINITY : 0.f);
        const float u = accept_uniform(p.seed, s_step, (uint32_t)rt);
        flag = fabsf(u - ratio) < kMargin;
        acc = u < ratio;
      } else {
        flag = (sz.x - sz.z) / fmaxf(1.f, fabsf(sz.x)) < kMargin;
        acc = d == __float_as_int(sz.y);
      }
    }
    const unsigned rej = __ballot_sync(0xffffffffu, !acc && lane < p.k);
    const int a = rej ? __ffs(rej) - 1 : p.k;
    // margins count for the decisions actually taken: drafts 1 .. a+1
    const unsigned flags = __ballot_sync(0xffffffffu, flag && lane <= a);
    if (lane == 0) {
      const float4 sz = n_rows > 0 ? s_rows[a] : make_float4(0.f, 1.f, 0.f, 0.f);
      const float4 sy = (n_rows > 0 && p.T > 0.f && a < p.k) ? s_rows[p.n_q + a]
                                                              : make_float4(0.f, 1.f, 0.f, 0.f);
      s_a = a;
      s_flag = flags != 0;
      s_mz = sz.x;
      s_isz = 1.f / sz.y;
      s_my = sy.x;
      s_isy = 1.f / sy.y;
      s_top1 = sz.x;
      s_arg = __float_as_int(sz.y);
      s_top2 = sz.z;
    }
  }
  __syncthreads();
  const int a = s_a;
  const uint32_t step = s_step;

  if (p.T == 0.f) {  // greedy: one CTA per sequence, no race
    if (threadIdx.x == 0) {
      int flag = s_flag;
      if ((s_top1 - s_top2) / fmaxf(1.f, fabsf(s_top1)) < kMargin) flag = 1;
      int32_t *o = p.out + (size_t)b * p.ld_o;
      for (int j = 0; j < p.n_q; ++j)
        o[j] = j < a ? p.drafts[(size_t)b * p.k + j] : (j == a ? s_arg : -1);
      p.n_acc[b] = a;
      if (p.margin) p.margin[b] = flag;
    }
    return;
  }

  // ---- exponential race over this CTA's chunk of the draw row
  const bool resid = a < p.k;
  const int rt = b * p.n_q + a;
  const float *zr = p.z + (size_t)rt * p.ld_t;
  const float *yr = resid ? p.y + ((size_t)b * p.k + a) * p.ld_d : nullptr;
  const float mz = s_mz, isz = s_isz, my = resid ? s_my : 0.f, isy = resid ? s_isy : 0.f;
  const int v0 = c * p.draw_chunk;
  const int v1 = min(p.V, v0 + p.draw_chunk);
  const int n4 = (v1 - v0) >> 2;
  Cand cr{-INFINITY, -INFINITY, -1}, cp{-INFINITY, -INFINITY, -1};
  // Keys in float32 with fast exp2 / log where the error (<~1e-6 absolute on a key, <~1e-6
  // relative on p and q) is far inside the 1e-4 margin below which a draw is flagged; the
  // log1p of the uniform stays accurate because small uniforms decide the winners.
  constexpr float L2E = 1.4426950408889634f;
  const bool unit_t = p.T == 1.f;
  const float mzl = mz * L2E, myl = my * L2E;
  const bool want_part = p.sout != nullptr;
  float pm = -INFINITY, ps = 0.f;
  for (int i = threadIdx.x; i < n4; i += kThreads) {
    const int v = v0 + 4 * i;
    const float4 z4 = __ldg(reinterpret_cast<const float4 *>(zr + v));
    float4 y4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (resid) y4 = __ldg(reinterpret_cast<const float4 *>(yr + v));
    const float zz[4] = {z4.x, z4.y, z4.z, z4.w};
    const float yy[4] = {y4.x, y4.y, y4.z, y4.w};
    float zt[4], w[4];
    bool any = false;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      zt[e] = unit_t ? zz[e] : zz[e] / p.T;
      w[e] = 0.f;
      if (resid) {
        const float yt = unit_t ? yy[e] : yy[e] / p.T;
        const float pv = ex2_approx(fmaf(zt[e], L2E, -mzl)) * isz;
        const float qv = ex2_approx(fmaf(yt, L2E, -myl)) * isy;
        w[e] = pv - qv;
      }
      any |= zt[e] != -INFINITY || w[e] > 0.f;
    }
    if (want_part) {  // running (max, sum exp(x - max)) of the drawn row's logits / T
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (zt[e] == -INFINITY) continue;
        if (zt[e] > pm) {
          ps = ps * exp2f((pm - zt[e]) * L2E) + 1.f;
          pm = zt[e];
        } else {
          ps += exp2f((zt[e] - pm) * L2E);
        }
      }
    }
    if (!any) continue;  // no token of the group can win either race: no uniforms needed
    float U[4];
    token_uniform_pair(p.seed, step, (uint32_t)rt, (uint32_t)p.purpose, (uint32_t)(v >> 1), U[0],
                       U[1]);
    token_uniform_pair(p.seed, step, (uint32_t)rt, (uint32_t)p.purpose, (uint32_t)(v >> 1) + 1u,
                       U[2], U[3]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lnE = __logf(neg_log1m(U[e]));  // E == 0 gives -inf: that token wins
      cand_push(cp, zt[e] == -INFINITY ? -INFINITY : zt[e] - lnE, v + e);
      if (resid) cand_push(cr, w[e] > 0.f ? __logf(w[e]) - lnE : -INFINITY, v + e);
    }
  }
  for (int off = 16; off > 0; off >>= 1) {
    const Cand o1 = cand_shfl(cp, off), o2 = cand_shfl(cr, off);
    cp = (lane & off) ? cand_merge(o1, cp) : cand_merge(cp, o1);
    cr = (lane & off) ? cand_merge(o2, cr) : cand_merge(cr, o2);
  }
  if (want_part) {
    for (int off = 16; off > 0; off >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, pm, off);
      const float s2 = __shfl_xor_sync(0xffffffffu, ps, off);
      ms_merge(pm, ps, m2, s2);
    }
  }
  if (lane == 0) {
    red[0][warp] = make_float4(cp.g1, __int_as_float(cp.v1), cp.g2, 0.f);
    red[1][warp] = make_float4(cr.g1, __int_as_float(cr.v1), cr.g2, 0.f);
    s_part[warp] = make_float2(pm, ps);
  }
  __syncthreads();
  if (want_part && threadIdx.x == 0) {
    float M = s_part[0].x, S = s_part[0].y;
    for (int w = 1; w < kThreads / 32; ++w) ms_merge(M, S, s_part[w].x, s_part[w].y);
    p.sout[(size_t)b * p.sld + c] = make_float2(M, S);
  }
  if (threadIdx.x == 0) {
    Cand tp{red[0][0].x, red[0][0].z, __float_as_int(red[0][0].y)};
    Cand tr{red[1][0].x, red[1][0].z, __float_as_int(red[1][0].y)};
    for (int w = 1; w < kThreads / 32; ++w) {
      tp = cand_merge(tp, Cand{red[0][w].x, red[0][w].z, __float_as_int(red[0][w].y)});
      tr = cand_merge(tr, Cand{red[1][w].x, red[1][w].z, __float_as_int(red[1][w].y)});
    }
    float4 *slot = p.cand + ((size_t)b * p.ndraw + c) * 2;
    slot[0] = make_float4(tp.g1, __int_as_float(tp.v1), tp.g2, 0.f);
    slot[1] = make_float4(tr.g1, __int_as_float(tr.v1), tr.g2, 0.f);
    __threadfence();
    const unsigned int ticket = atomicAdd(&p.counters[b], 1u);
    s_last = ticket == (unsigned int)(p.ndraw - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // ---- last CTA of the sequence: merge the chunk winners (order-independent: ties go to the
  // lower token id), one warp
  if (threadIdx.x >= 32) return;
  const volatile float4 *cv = reinterpret_cast<const volatile float4 *>(p.cand) +
                              (size_t)b * p.ndraw * 2;
  Cand tp{-INFINITY, -INFINITY, -1}, tr{-INFINITY, -INFINITY, -1};
  for (int cc = lane; cc < p.ndraw; cc += 32) {
    const float a0x = cv[2 * cc].x, a0y = cv[2 * cc].y, a0z = cv[2 * cc].z;
    const float a1x = cv[2 * cc + 1].x, a1y = cv[2 * cc + 1].y, a1z = cv[2 * cc + 1].z;
    tp = cand_merge(tp, Cand{a0x, a0z, __float_as_int(a0y)});
    tr = cand_merge(tr, Cand{a1x, a1z, __float_as_int(a1y)});
  }
  for (int off = 16; off > 0; off >>= 1) {
    tp = cand_merge(tp, cand_shfl(tp, off));
    tr = cand_merge(tr, cand_shfl(tr, off));
  }
  if (lane != 0) return;
  const Cand &w = (resid && tr.v1 >= 0 && tr.g1 > -INFINITY) ? tr : tp;
  int flag = s_flag;
  if (w.g1 - w.g2 < kMargin) flag = 1;
  int32_t *o = p.out + (size_t)b * p.ld_o;
  for (int j = 0; j < p.n_q; ++j)
    o[j] = j < a ? p.drafts[(size_t)b * p.k + j] : (j == a ? w.v1 : -1);
  p.n_acc[b] = a;
  if (p.margin) p.margin[b] = flag;
  p.counters[b] = 0u;
}

// Zeroes the per-sequence tickets of the draw (plain draws, which skip the statistics pass
// that otherwise clears them).
__global__ void clear_tickets_kernel(unsigned int *counters, int B) {
  pdl_wait();
  for (int b = threadIdx.x; b < B; b += blockDim.x) counters[b] = 0u;
}

static int ndraw_of(int B, int V);

static sd_status validate(const sd_accept_desc *d) {
  if (!d) return SD_ERR_INVALID_ARG;
  if (d->batch < 1 || d->k < 0 || d->k > 15 || d->vocab < 1) return SD_ERR_INVALID_ARG;
  if (!(d->temperature >= 0.f) || d->temperature > 1e30f) return SD_ERR_INVALID_ARG;
  if (d->purpose < 1) return SD_ERR_INVALID_ARG;
  const int ldt = d->ld_target ? d->ld_target : d->vocab;
  const int ldd = d->ld_draft ? d->ld_draft : d->vocab;
  const int ldo = d->ld_out ? d->ld_out : d->k + 1;
  if (ldt < d->vocab || ldd < d->vocab || ldo < d->k + 1) return SD_ERR_INVALID_ARG;
  if (d->vocab % 4 || ldt % 4 || ldd % 4) return SD_ERR_UNSUPPORTED;
  if (d->target_stats &&
      (d->target_stats_slots < 1 ||
       (d->ld_target_stats != 0 && d->ld_target_stats < d->target_stats_slots)))
    return SD_ERR_INVALID_ARG;
  if (d->draft_stats &&
      (d->draft_stats_slots < 1 ||
       (d->ld_draft_stats != 0 && d->ld_draft_stats < d->draft_stats_slots)))
    return SD_ERR_INVALID_ARG;
  if (d->stats_out) {
    if (d->k != 0 || !(d->temperature > 0.f)) return SD_ERR_INVALID_ARG;
    if (d->ld_stats_out != 0 && d->ld_stats_out < ndraw_of(d->batch, d->vocab))
      return SD_ERR_INVALID_ARG;
  }
  return SD_OK;
}

static int nchunks_of(int V) { return (V + kChunk - 1) / kChunk; }

// Tokens per CTA of the statistics pass: kChunk, or more (multiples of 1024) when the rows
// times kChunk-token chunks would not fit in one wave of CTAs.  Never more chunks per row than
// nchunks_of(V), which sizes the workspace.
static int stats_chunk_of(int rows, int V) {
  static int occ_cache[64];
  int dev = 0;
  cudaGetDevice(&dev);
  int occ = dev < 64 ? occ_cache[dev] : 0;
  if (occ <= 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, accept_stats_kernel, kThreads, 0) !=
            cudaSuccess ||
        occ <= 0)
      occ = 1;
    if (dev < 64) occ_cache[dev] = occ;
  }
  const int sms = sm_count();
  const long long slots = (long long)occ * (sms > 0 ? sms : 148);
  long long n = slots / (rows > 0 ? rows : 1);
  if (n < 1) n = 1;
  if (n > nchunks_of(V)) n = nchunks_of(V);
  int chunk = (int)((V + n - 1) / n);
  chunk = (chunk + 1023) / 1024 * 1024;
  return chunk < kChunk ? kChunk : chunk;
}
// Tokens per draw CTA: the race of one sequence is split so that all B sequences together give
// about one wave of CTAs (the per-CTA chain of dependent memory round trips, not the token work,
// dominates at small B); multiples of 1024 tokens.
static int draw_chunk_of(int B, int V) {
  int per_seq = kDrawSlots / (B > 0 ? B : 1);
  if (per_seq < 1) per_seq = 1;
  int chunk = (V + per_seq - 1) / per_seq;
  chunk = (chunk + 1023) / 1024 * 1024;
  return chunk;
}
static int ndraw_of(int B, int V) {
  const int c = draw_chunk_of(B, V);
  return (V + c - 1) / c;
}

static size_t ws_size(const sd_accept_desc *d) {
  if (validate(d) != SD_OK) return 0;
  const size_t nc = nchunks_of(d->vocab);
  const size_t rows = (size_t)d->batch * (d->k + 1) + (size_t)d->batch * d->k;
  return round_up(rows * nc * 16, 256) +
         round_up((size_t)d->batch * ndraw_of(d->batch, d->vocab) * 32, 256) +
         round_up((size_t)d->batch * 4, 256);
}

}  // namespace acc
}  // namespace sdv

extern "C" {

size_t sd_accept_workspace_size(const sd_accept_desc *desc) { return sdv::acc::ws_size(desc); }

int sd_accept_stats_slots(const sd_accept_desc *desc) {
  if (sdv::acc::validate(desc) != SD_OK || desc->k != 0 || !(desc->temperature > 0.f)) return 0;
  return sdv::acc::ndraw_of(desc->batch, desc->vocab);
}

sd_status sd_accept(const sd_accept_desc *desc, const float *target_logits,
                    const float *draft_logits, const int32_t *draft_tokens,
                    int32_t *n_accepted, int32_t *out_tokens, int32_t *margin_flags,
                    void *ws, size_t ws_bytes, sd_stream stream) {
  using namespace sdv;
  using namespace sdv::acc;
  sd_status s = validate(desc);
  if (s != SD_OK) return s;
  const bool sampling = desc->temperature > 0.f;
  if (!target_logits || !n_accepted || !out_tokens) return SD_ERR_INVALID_ARG;
  if (desc->k > 0 && !draft_tokens) return SD_ERR_INVALID_ARG;
  if (sampling && desc->k > 0 && !draft_logits) return SD_ERR_INVALID_ARG;
  if (!aligned16(target_logits) || (sampling && desc->k > 0 && !aligned16(draft_logits)))
    return SD_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < ws_size(desc)) return SD_ERR_WORKSPACE;
  Params p{};
  p.B = desc->batch;
  p.k = desc->k;
  p.V = desc->vocab;
  p.n_q = desc->k + 1;
  p.ld_t = desc->ld_target ? desc->ld_target : desc->vocab;
  p.ld_d = desc->ld_draft ? desc->ld_draft : desc->vocab;
  p.ld_o = desc->ld_out ? desc->ld_out : desc->k + 1;
  p.purpose = desc->purpose;
  p.draw_chunk = draw_chunk_of(desc->batch, desc->vocab);
  p.ndraw = ndraw_of(desc->batch, desc->vocab);
  p.rows_t = p.B * p.n_q;
  p.rows_total = p.rows_t + (sampling ? p.B * p.k : 0);
  // producer partials (sampling only; the greedy rule needs the top two of each row)
  if (sampling && desc->target_stats) {
    p.tstats = reinterpret_cast<const float2 *>(desc->target_stats);
    p.tslots = desc->target_stats_slots;
    p.tld = desc->ld_target_stats ? desc->ld_target_stats : desc->target_stats_slots;
  }
  if (sampling && p.k > 0 && desc->draft_stats) {
    p.dstats = reinterpret_cast<const float2 *>(desc->draft_stats);
    p.dslots = desc->draft_stats_slots;
    p.dld = desc->ld_draft_stats ? desc->ld_draft_stats : desc->draft_stats_slots;
  }
  // rows the statistics pass still computes: target rows, then draft rows
  const bool need_t = !(sampling && (p.k == 0 || p.tstats != nullptr));
  const bool need_d = sampling && p.k > 0 && p.dstats == nullptr;
  p.stats_row0 = need_t ? 0 : p.rows_t;
  p.stats_rows = (need_t ? p.rows_t : 0) + (need_d ? p.rows_total - p.rows_t : 0);
  p.stats_chunk = stats_chunk_of(p.stats_rows > 0 ? p.stats_rows : 1, desc->vocab);
  p.nchunks = (desc->vocab + p.stats_chunk - 1) / p.stats_chunk;
  p.T = desc->temperature;
  p.seed = desc->seed;
  p.step = desc->step;
  p.step_ptr = reinterpret_cast<const unsigned long long *>(desc->step_ptr);
  p.z = target_logits;
  p.y = draft_logits;
  p.drafts = draft_tokens;
  p.n_acc = n_accepted;
  p.out = out_tokens;
  p.margin = margin_flags;
  if (desc->stats_out) {
    p.sout = reinterpret_cast<float2 *>(desc->stats_out);
    p.sld = desc->ld_stats_out ? desc->ld_stats_out : p.ndraw;
  }
  const size_t rows = (size_t)p.B * (p.k + 1) + (size_t)p.B * p.k;
  uint8_t *w8 = reinterpret_cast<uint8_t *>(ws);
  p.stats = reinterpret_cast<float4 *>(w8);
  w8 += round_up(rows * p.nchunks * 16, 256);
  p.cand = reinterpret_cast<float4 *>(w8);
  w8 += round_up((size_t)p.B * p.ndraw * 32, 256);
  p.counters = reinterpret_cast<unsigned int *>(w8);
  p.status = device_status_word();
  cudaStream_t st = (cudaStream_t)stream;
  if (p.stats_rows == 0) {
    // every row's statistics come from elsewhere (a plain draw needs none): only the
    // per-sequence tickets need clearing (a one-block kernel: in a CUDA graph it costs less
    // than a memset node)
    if (launch(clear_tickets_kernel, dim3(1), dim3(kThreads), 0, st, p.counters, p.B) !=
        cudaSuccess)
      return SD_ERR_CUDA;
  } else if (launch(accept_stats_kernel, dim3(p.stats_rows, p.nchunks), dim3(kThreads), 0, st,
                    p) != cudaSuccess) {
    return SD_ERR_CUDA;
  }
  return cuda_status(
      launch(accept_draw_kernel, dim3(p.B, sampling ? p.ndraw : 1), dim3(kThreads), 0, st, p));
}

}  // extern "C"

// ----------------------------------------------------------------------------- no-allocation
// sd_accept_noalloc: the same acceptance step for callers that cannot allocate device memory
// themselves -- for example code running where a device allocation would synchronise or is
// forbidden (inside a real-time serving loop with a fixed memory budget, or a host framework
// that hands out only its own buffers).  The scratch lives in a fixed array compiled into this
// library; every GPU that loads the library keeps it until the process exits.

namespace sdv {
namespace acc {

static __device__ __align__(256) unsigned char g_accept_noalloc_scratch[SD_ACCEPT_NOALLOC_MAX_SCRATCH];

// Device address of the scratch array on the current device, looked up once per device.  A
// symbol's host-side name is not a device address, so it is never passed to a kernel directly.
static void *noalloc_scratch() {
  static std::mutex mu;
  static void *addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_accept_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace acc
}  // namespace sdv

extern "C" sd_status sd_accept_noalloc(const sd_accept_desc *desc, const float *target_logits,
                                       const float *draft_logits, const int32_t *draft_tokens,
                                       int32_t *n_accepted, int32_t *out_tokens,
                                       int32_t *margin_flags, sd_stream stream) {
  const sd_status v = sdv::acc::validate(desc);
  if (v != SD_OK) return v;
  if (sd_accept_workspace_size(desc) > (size_t)SD_ACCEPT_NOALLOC_MAX_SCRATCH)
    return SD_ERR_WORKSPACE;
  void *scratch = sdv::acc::noalloc_scratch();
  if (scratch == nullptr) return SD_ERR_CUDA;
  // The per-sequence counters in the scratch are cleared at the start of every call (by the
  // statistics kernel, or a one-block kernel for a plain draw), so the array's leftover
  // contents from an earlier call do not matter.
  return sd_accept(desc, target_logits, draft_logits, draft_tokens, n_accepted, out_tokens,
                   margin_flags, scratch, (size_t)SD_ACCEPT_NOALLOC_MAX_SCRATCH, stream);
}
