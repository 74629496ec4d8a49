// Lossless acceptance of k drafts, correction / bonus draw, greedy rule (sm_100a).
//
// The rule (pages cite Leviathan et al. for it: Google blog translation, section "how
// speculative decoding works"; property stated in "Gemma 4 MTP: drafter drafts, target
// verifies", section "basic structure of speculative decoding"): accept d_i iff
// u_i < p_i(d_i) / q_i(d_i); at the first rejection emit x ~ norm(max(0, p_i - q_i)); if all
// are accepted emit the bonus x ~ p_{k+1}.  T = 0: accept iff d_i == argmax, emit argmax.
//
// Two kernels:
//  1. accept_decide: one thread-block cluster per sequence.  CTA c of the cluster streams
//     token slice c of every logit row the sequence needs (its k+1 target rows and, for
//     T > 0, its k draft rows) from HBM into shared memory with bulk copies (a 3-stage ring)
//     and reduces each row slice: online max / sum of exp(x / T) (T > 0) or the top two values
//     and the argmax (T = 0).  CTA 0 merges the slices' partials through distributed shared
//     memory in rank order and takes the acceptance decisions; at T = 0 it writes the outputs,
//     at T > 0 it writes the sequence's decision record (accepted count, margin flag, the
//     normalisers of the draw row) for the draw kernel.
//  2. accept_draw: one CTA per (sequence, token chunk), one wave of CTAs.  Exponential race of
//     the draw row over the chunk: key_v = ln w_v - ln(-ln(1 - V_v)), V_v the token's Philox
//     uniform, for the residual weights max(0, p - q) and for p (the bonus draw, and the
//     fallback when the residual is empty).  Each race keeps its winner, the winner's lowest
//     possible key and the highest possible key of every other token under the float32 error
//     model of the margin rule.  The last CTA of a sequence (atomic ticket; no waiting) merges
//     the chunk winners (lowest token id first on equal keys) and writes the outputs.
//  A plain draw (k = 0, T > 0, the drafter sampling its own token) runs the draw kernel alone:
//  its race keys are unnormalised logits / T, so no row statistics are needed.
#include <cfloat>

#include "common.cuh"
#include "host.cuh"
#include "philox.cuh"

namespace sdv {
namespace acc {

constexpr int kDecideThreads = 512;
constexpr int kPiece = 16384;       // floats per bulk copy of the decision pass (64 KB)
constexpr int kStages = 3;          // bulk-copy ring depth of the decision pass
constexpr int kMaxRows = 31;        // rows per sequence: 2k + 1 with k <= 15
constexpr int kDrawSlots = 592;     // draw CTAs aimed at: one wave at 4 CTAs on each of 148 SMs
constexpr int kDrawThreads = 256;
constexpr float kMargin = 1e-4f;    // spec margin on |u - p/q|; also for draws, argmaxes
constexpr float kRelP = 1e-5f;      // float32 error bound assumed on a probability p_v or q_v
constexpr float kAbsKey = 1e-5f;    // float32 error bound assumed on ln E_v and z_v / T

// Decision record of one sequence (T > 0): written by the decision kernel, read by the draw.
struct Record {
  int a;          // accepted drafts
  int flag;       // an acceptance test within the margin
  uint32_t step;  // counter step of the draws
  int pad;
  float mz, isz;  // max and 1 / sum exp of row a of the target logits / T
  float my, isy;  // the same for draft row a (a < k)
};

struct Params {
  int B, k, V, n_q, ld_t, ld_d, ld_o, purpose;
  int rps;           // rows per sequence read by the decision pass
  int cl;            // CTAs per sequence (the cluster) of the decision pass
  int slice;         // tokens per CTA of the decision pass (a multiple of 4)
  int npieces;       // bulk copies per row slice
  int ndraw, draw_chunk;
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
  Record *rec;             // [B]
  float4 *cand;            // [B][ndraw][3]
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

// ------------------------------------------------------------------ top two (greedy rule)

struct Top2 {  // best and runner-up value, best token id
  float g1, g2;
  int v1;
};

__device__ __forceinline__ void top2_push(Top2 &c, float g, int v) {
  // tokens arrive in increasing v per thread; strict > keeps the lowest id on ties
  if (g > c.g1) {
    c.g2 = c.g1;
    c.g1 = g;
    c.v1 = v;
  } else if (g > c.g2) {
    c.g2 = g;
  }
}

__device__ __forceinline__ Top2 top2_merge(const Top2 &a, const Top2 &b) {
  // on equal values the lower token id wins, whatever the order of a and b
  Top2 r;
  if (b.g1 > a.g1 || (b.g1 == a.g1 && b.v1 >= 0 && (a.v1 < 0 || b.v1 < a.v1))) {
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

__device__ __forceinline__ Top2 top2_shfl(const Top2 &c, int off) {
  Top2 o;
  o.g1 = __shfl_xor_sync(0xffffffffu, c.g1, off);
  o.g2 = __shfl_xor_sync(0xffffffffu, c.g2, off);
  o.v1 = __shfl_xor_sync(0xffffffffu, c.v1, off);
  return o;
}

// ------------------------------------------------------------------ race candidates

// Winner of an exponential race with the bounds of the margin rule: the winner's key g1, its
// lowest possible key lo1 and highest possible key hi1, and hi2, the highest possible key of
// every other token seen.  The draw is flagged when hi2 > lo1 - margin: some other token might
// have won under float32 error.
struct Race {
  float g1, lo1, hi1, hi2;
  int v1;
};

__device__ __forceinline__ Race race_empty() { return Race{-INFINITY, -INFINITY, -INFINITY, -INFINITY, -1}; }

__device__ __forceinline__ void race_push(Race &c, float g, float lo, float hi, int v) {
  if (g > c.g1) {  // tokens arrive in increasing v per thread: ties keep the lower id
    c.hi2 = fmaxf(c.hi2, c.hi1);
    c.g1 = g;
    c.lo1 = lo;
    c.hi1 = hi;
    c.v1 = v;
  } else {
    c.hi2 = fmaxf(c.hi2, hi);
  }
}

__device__ __forceinline__ Race race_merge(const Race &a, const Race &b) {
  const bool bw = b.g1 > a.g1 || (b.g1 == a.g1 && b.v1 >= 0 && (a.v1 < 0 || b.v1 < a.v1));
  const Race &w = bw ? b : a;
  const Race &l = bw ? a : b;
  Race r = w;
  r.hi2 = fmaxf(w.hi2, fmaxf(l.hi1, l.hi2));
  return r;
}

__device__ __forceinline__ Race race_shfl(const Race &c, int off) {
  Race o;
  o.g1 = __shfl_xor_sync(0xffffffffu, c.g1, off);
  o.lo1 = __shfl_xor_sync(0xffffffffu, c.lo1, off);
  o.hi1 = __shfl_xor_sync(0xffffffffu, c.hi1, off);
  o.hi2 = __shfl_xor_sync(0xffffffffu, c.hi2, off);
  o.v1 = __shfl_xor_sync(0xffffffffu, c.v1, off);
  return o;
}

__device__ __forceinline__ bool race_flag(const Race &r) { return r.hi2 > r.lo1 - kMargin; }

// (max, sum exp(x - max)) pairs
__device__ __forceinline__ void ms_merge(float &m, float &s, float m2, float s2) {
  const float mm = fmaxf(m, m2);
  if (mm == -INFINITY) return;
  s = s * expf(m - mm) + s2 * expf(m2 - mm);
  m = mm;
}

__device__ __forceinline__ const float *seq_row(const Params &p, int b, int ri) {
  return ri < p.n_q ? p.z + (size_t)(b * p.n_q + ri) * p.ld_t
                    : p.y + (size_t)(b * p.k + ri - p.n_q) * p.ld_d;
}

__device__ __forceinline__ uint32_t counter_step(const Params &p) {
  return (uint32_t)(p.step + (p.step_ptr != nullptr ? *p.step_ptr : 0ull));
}

// ------------------------------------------------------------------ decision kernel

__global__ void __launch_bounds__(kDecideThreads, 1) accept_decide_kernel(const Params p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float *ring = reinterpret_cast<float *>(smem_raw);  // [kStages][piece]
  __shared__ uint64_t full[kStages];
  __shared__ float4 s_wpart[kMaxRows][kDecideThreads / 32];
  __shared__ float4 s_part[kMaxRows];   // this CTA's slice partial of each row
  __shared__ float4 s_row[kMaxRows];    // merged rows (CTA 0)
  __shared__ int s_abort;
  __shared__ uint32_t s_step;
  pdl_wait();
  const uint32_t rank = cluster_ctarank();
  const int ncl = p.cl;       // CTAs per sequence: the cluster
  const int b = blockIdx.x / ncl;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = blockDim.x >> 5;
  const int v0 = (int)rank * p.slice;
  const int v1 = min(p.V, v0 + p.slice);
  const int n = max(0, v1 - v0);
  const int piece = (n + p.npieces - 1) / p.npieces;
  const int piece4 = (piece + 3) & ~3;
  const int units = p.rps * p.npieces;
  const bool sampling = p.T > 0.f;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
    s_abort = 0;
    if (rank == 0) s_step = counter_step(p);
  }
  __syncthreads();
  // unit u = (row u / npieces, piece u % npieces); its tokens [v0 + piece4 * pc, ...)
  auto unit_range = [&](int u, int &ri, int &t0, int &cnt) {
    ri = u / p.npieces;
    const int pc = u - ri * p.npieces;
    t0 = v0 + pc * piece4;
    cnt = max(0, min(v1, t0 + piece4) - t0);
  };
  auto issue = [&](int u) {
    int ri, t0, cnt;
    unit_range(u, ri, t0, cnt);
    const int s = u % kStages;
    if (cnt > 0) {
      mbar_arrive_expect_tx(&full[s], (uint32_t)cnt * 4u);
      bulk_load(ring + (size_t)s * piece4, seq_row(p, b, ri) + t0, (uint32_t)cnt * 4u, &full[s]);
    } else {
      mbar_arrive(&full[s]);
    }
  };
  if (tid == 0)
    for (int u = 0; u < kStages && u < units; ++u) issue(u);

  constexpr float L2E = 1.4426950408889634f;
  const float inv_t = sampling ? 1.f / p.T : 1.f;
  // per-warp partial of the current row, merged over its pieces
  float wm = -INFINITY, ws = 0.f;
  Top2 wt{-INFINITY, -INFINITY, -1};
  int last_issued = min(kStages, units) - 1;  // (thread 0) the latest unit copied
  for (int u = 0; u < units; ++u) {
    const int s = u % kStages;
    int ri, t0, cnt;
    unit_range(u, ri, t0, cnt);
    if (s_abort == 0 && !mbar_wait(&full[s], (u / kStages) & 1, &s_abort)) {
      record_status(p.status, SD_ERR_TIMEOUT);
      s_abort = 1;
    }
    if (s_abort == 0) {
      const float *buf = ring + (size_t)s * piece4;
      const int n4 = cnt >> 2;
      const float4 *buf4 = reinterpret_cast<const float4 *>(buf);
      if (sampling) {
        float m = -INFINITY, sm = 0.f;
        for (int i = tid; i < n4; i += blockDim.x) {
          float4 x = buf4[i];
          if (p.T != 1.f) x = make_float4(x.x * inv_t, x.y * inv_t, x.z * inv_t, x.w * inv_t);
          const float mb = fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w));
          if (mb == -INFINITY) continue;
          if (mb > m) {
            sm *= exp2f((m - mb) * L2E);
            m = mb;
          }
          sm += (exp2f((x.x - m) * L2E) + exp2f((x.y - m) * L2E)) +
                (exp2f((x.z - m) * L2E) + exp2f((x.w - m) * L2E));
        }
        for (int off = 16; off > 0; off >>= 1) {
          const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
          const float s2 = __shfl_xor_sync(0xffffffffu, sm, off);
          ms_merge(m, sm, m2, s2);
        }
        ms_merge(wm, ws, m, sm);
      } else {
        Top2 c{-INFINITY, -INFINITY, -1};
        for (int i = tid; i < n4; i += blockDim.x) {
          const float4 x = buf4[i];
          const int v = t0 + 4 * i;
          top2_push(c, x.x, v);
          top2_push(c, x.y, v + 1);
          top2_push(c, x.z, v + 2);
          top2_push(c, x.w, v + 3);
        }
        for (int off = 16; off > 0; off >>= 1) c = top2_merge(c, top2_shfl(c, off));
        wt = top2_merge(wt, c);
      }
    }
    const bool row_end = (u + 1) % p.npieces == 0;
    if (row_end && lane == 0) {
      s_wpart[ri][warp] = sampling ? make_float4(wm, ws, 0.f, 0.f)
                                   : make_float4(wt.g1, __int_as_float(wt.v1), wt.g2, 0.f);
    }
    if (row_end) {
      wm = -INFINITY;
      ws = 0.f;
      wt = Top2{-INFINITY, -INFINITY, -1};
    }
    __syncthreads();  // every thread is done with stage s: refill it
    if (tid == 0 && u + kStages < units && s_abort == 0) {
      issue(u + kStages);
      last_issued = u + kStages;
    }
  }
  if (s_abort != 0 && tid == 0) {
    // drain the copies still in flight (the latest one per stage) before the shared memory is
    // released
    for (int j = max(0, last_issued - kStages + 1); j <= last_issued; ++j)
      mbar_wait_timed(&full[j % kStages], (j / kStages) & 1);
  }
  // this CTA's partial of each row (warps merged in order)
  if (tid < p.rps) {
    float4 r = s_wpart[tid][0];
    for (int w = 1; w < nwarps; ++w) {
      const float4 o = s_wpart[tid][w];
      if (sampling) {
        ms_merge(r.x, r.y, o.x, o.y);
      } else {
        const Top2 t = top2_merge(Top2{r.x, r.z, __float_as_int(r.y)},
                                  Top2{o.x, o.z, __float_as_int(o.y)});
        r = make_float4(t.g1, __int_as_float(t.v1), t.g2, 0.f);
      }
    }
    s_part[tid] = r;
  }
  cluster_sync();  // every CTA's partials are visible to CTA 0
  if (rank == 0) {
    // merge the slices of row w in rank order (one warp per row)
    for (int ri = warp; ri < p.rps; ri += nwarps) {
      float4 v = lane < ncl ? ld_dsmem_f4(dsmem_addr(smem_u32(&s_part[ri]), lane))
                            : (sampling ? make_float4(-INFINITY, 0.f, 0.f, 0.f)
                                        : make_float4(-INFINITY, __int_as_float(-1), -INFINITY,
                                                      0.f));
      if (sampling) {
        for (int off = 16; off > 0; off >>= 1) {
          const float m2 = __shfl_xor_sync(0xffffffffu, v.x, off);
          const float s2 = __shfl_xor_sync(0xffffffffu, v.y, off);
          ms_merge(v.x, v.y, m2, s2);
        }
      } else {
        Top2 t{v.x, v.z, __float_as_int(v.y)};
        for (int off = 16; off > 0; off >>= 1) t = top2_merge(t, top2_shfl(t, off));
        v = make_float4(t.g1, __int_as_float(t.v1), t.g2, 0.f);
      }
      if (lane == 0) s_row[ri] = v;
    }
  }
  cluster_sync();  // CTA 0 has read the other CTAs' shared memory: they may exit
  if (rank != 0 || warp != 0) return;

  // ---- decisions (one warp): lane i-1 tests draft i; the first rejection stops the scan
  const uint32_t step = s_step;
  bool acc = true;
  int flag = 0;
  if (lane < p.k) {
    const int d = p.drafts[(size_t)b * p.k + lane];
    const int rt = b * p.n_q + lane;
    const float4 sz = s_row[lane];
    if (d < 0 || d >= p.V) {
      record_status(p.status, SD_ERR_DEVICE);
      acc = false;
    } else if (sampling) {
      const float4 sy = s_row[p.n_q + lane];
      const float pd = expf(p.z[(size_t)rt * p.ld_t + d] * inv_t - sz.x) / sz.y;
      const float qd = expf(p.y[((size_t)b * p.k + lane) * p.ld_d + d] * inv_t - sy.x) / sy.y;
      const float ratio = qd > 0.f ? pd / qd : (pd > 0.f ? INFINITY : 0.f);
      const float u = accept_uniform(p.seed, step, (uint32_t)rt);
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
  const int any_flag = __ballot_sync(0xffffffffu, flag && lane <= a) != 0;
  if (lane != 0) return;
  const float4 sz = s_row[a];
  if (!sampling) {
    int f = any_flag;
    if ((sz.x - sz.z) / fmaxf(1.f, fabsf(sz.x)) < kMargin) f = 1;
    int32_t *o = p.out + (size_t)b * p.ld_o;
    for (int j = 0; j < p.n_q; ++j)
      o[j] = j < a ? p.drafts[(size_t)b * p.k + j] : (j == a ? __float_as_int(sz.y) : -1);
    p.n_acc[b] = a;
    if (p.margin) p.margin[b] = f;
    return;
  }
  const float4 sy = a < p.k ? s_row[p.n_q + a] : make_float4(0.f, 1.f, 0.f, 0.f);
  Record r;
  r.a = a;
  r.flag = any_flag;
  r.step = step;
  r.pad = 0;
  r.mz = sz.x;
  r.isz = 1.f / sz.y;
  r.my = sy.x;
  r.isy = 1.f / sy.y;
  p.rec[b] = r;
  p.counters[b] = 0u;  // tickets of the draw kernel
}

// ------------------------------------------------------------------ draw kernel

__global__ void __launch_bounds__(kDrawThreads) accept_draw_kernel(const Params p) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x, c = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __shared__ Record s_rec;
  __shared__ Race s_red[2][kDrawThreads / 32];
  __shared__ int s_last;

  if (threadIdx.x == 0) {
    if (p.k == 0) {  // plain draw: no decisions, unnormalised keys
      s_rec = Record{0, 0, counter_step(p), 0, 0.f, 1.f, 0.f, 1.f};
    } else {
      s_rec = p.rec[b];
    }
  }
  __syncthreads();
  const int a = s_rec.a;
  const uint32_t step = s_rec.step;
  const bool resid = a < p.k;
  const int rt = b * p.n_q + a;
  const float *zr = p.z + (size_t)rt * p.ld_t;
  const float *yr = resid ? p.y + ((size_t)b * p.k + a) * p.ld_d : nullptr;
  const float isz = s_rec.isz, isy = s_rec.isy;
  const int v0 = c * p.draw_chunk;
  const int v1 = min(p.V, v0 + p.draw_chunk);
  const int n4 = max(0, v1 - v0) >> 2;
  Race cp = race_empty(), cr = race_empty();
  // Keys in float32 with fast exp2 / log where the error (<~1e-6 absolute on a key, <~1e-6
  // relative on p and q) is far inside the error model the bounds assume (1e-5); the log1p of
  // the uniform stays accurate because small uniforms decide the winners.
  constexpr float L2E = 1.4426950408889634f;
  const bool unit_t = p.T == 1.f;
  const float inv_t = 1.f / p.T;
  const float mzl = s_rec.mz * L2E, myl = s_rec.my * L2E;
  for (int i = threadIdx.x; i < n4; i += kDrawThreads) {
    const int v = v0 + 4 * i;
    const float4 z4 = __ldg(reinterpret_cast<const float4 *>(zr + v));
    float4 y4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (resid) y4 = __ldg(reinterpret_cast<const float4 *>(yr + v));
    const float zz[4] = {z4.x, z4.y, z4.z, z4.w};
    const float yy[4] = {y4.x, y4.y, y4.z, y4.w};
    float zt[4], w[4], sl[4];
    bool any = false;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      zt[e] = unit_t ? zz[e] : zz[e] * inv_t;
      w[e] = 0.f;
      sl[e] = 0.f;
      if (resid) {
        const float yt = unit_t ? yy[e] : yy[e] * inv_t;
        const float pv = ex2_approx(fmaf(zt[e], L2E, -mzl)) * isz;
        const float qv = ex2_approx(fmaf(yt, L2E, -myl)) * isy;
        w[e] = fmaxf(pv - qv, 0.f);
        sl[e] = kRelP * (pv + qv);
      }
      any |= zt[e] != -INFINITY || w[e] + sl[e] > 0.f;
    }
    if (!any) continue;  // no token of the group has any weight: no uniforms needed
    float U[4];
    token_uniform_pair(p.seed, step, (uint32_t)rt, (uint32_t)p.purpose, (uint32_t)(v >> 1), U[0],
                       U[1]);
    token_uniform_pair(p.seed, step, (uint32_t)rt, (uint32_t)p.purpose, (uint32_t)(v >> 1) + 1u,
                       U[2], U[3]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lnE = __logf(neg_log1m(U[e]));  // E == 0 gives -inf: that token wins
      if (zt[e] != -INFINITY) {
        const float g = zt[e] - lnE;
        const float err = kAbsKey * (1.f + fabsf(zt[e]));
        race_push(cp, g, g - err, g + err, v + e);
      }
      if (resid && w[e] + sl[e] > 0.f) {
        const float hi = __logf(w[e] + sl[e]) - lnE + kAbsKey;
        const float g = w[e] > 0.f ? __logf(w[e]) - lnE : -INFINITY;
        if (g > cr.g1) {
          const float wl = w[e] - sl[e];
          race_push(cr, g, wl > 0.f ? __logf(wl) - lnE - kAbsKey : -INFINITY, hi, v + e);
        } else {
          cr.hi2 = fmaxf(cr.hi2, hi);
        }
      }
    }
  }
  for (int off = 16; off > 0; off >>= 1) {
    const Race o1 = race_shfl(cp, off);
    cp = (lane & off) ? race_merge(o1, cp) : race_merge(cp, o1);
    if (resid) {
      const Race o2 = race_shfl(cr, off);
      cr = (lane & off) ? race_merge(o2, cr) : race_merge(cr, o2);
    }
  }
  if (lane == 0) {
    s_red[0][warp] = cp;
    s_red[1][warp] = cr;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    Race tp = s_red[0][0], tr = s_red[1][0];
    for (int w = 1; w < kDrawThreads / 32; ++w) {
      tp = race_merge(tp, s_red[0][w]);
      tr = race_merge(tr, s_red[1][w]);
    }
    float4 *slot = p.cand + ((size_t)b * p.ndraw + c) * 3;
    slot[0] = make_float4(tp.g1, tp.lo1, tp.hi1, tp.hi2);
    slot[1] = make_float4(tr.g1, tr.lo1, tr.hi1, tr.hi2);
    slot[2] = make_float4(__int_as_float(tp.v1), __int_as_float(tr.v1), 0.f, 0.f);
    __threadfence();
    const unsigned int ticket = atomicAdd(&p.counters[b], 1u);
    s_last = ticket == (unsigned int)(p.ndraw - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // ---- last CTA of the sequence: merge the chunk winners (order-independent: equal keys go to
  // the lower token id), one warp
  if (threadIdx.x >= 32) return;
  const volatile float4 *cv = reinterpret_cast<const volatile float4 *>(p.cand) +
                              (size_t)b * p.ndraw * 3;
  Race tp = race_empty(), tr = race_empty();
  for (int cc = lane; cc < p.ndraw; cc += 32) {
    const float4 a0 = make_float4(cv[3 * cc].x, cv[3 * cc].y, cv[3 * cc].z, cv[3 * cc].w);
    const float4 a1 =
        make_float4(cv[3 * cc + 1].x, cv[3 * cc + 1].y, cv[3 * cc + 1].z, cv[3 * cc + 1].w);
    const float ix = cv[3 * cc + 2].x, iy = cv[3 * cc + 2].y;
    tp = race_merge(tp, Race{a0.x, a0.y, a0.z, a0.w, __float_as_int(ix)});
    tr = race_merge(tr, Race{a1.x, a1.y, a1.z, a1.w, __float_as_int(iy)});
  }
  for (int off = 16; off > 0; off >>= 1) {
    tp = race_merge(tp, race_shfl(tp, off));
    tr = race_merge(tr, race_shfl(tr, off));
  }
  if (lane != 0) return;
  // the residual race unless every residual weight came out 0 (then p, and the draw is flagged:
  // a residual too small for float32 may still be positive)
  const bool use_r = resid && tr.v1 >= 0;
  const Race &w = use_r ? tr : tp;
  int flag = s_rec.flag;
  if (race_flag(w) || (resid && !use_r)) flag = 1;
  int32_t *o = p.out + (size_t)b * p.ld_o;
  for (int j = 0; j < p.n_q; ++j)
    o[j] = j < a ? p.drafts[(size_t)b * p.k + j] : (j == a ? w.v1 : -1);
  p.n_acc[b] = a;
  if (p.margin) p.margin[b] = flag;
  p.counters[b] = 0u;
}

// Zeroes the per-sequence tickets of the draw (plain draws, which have no decision pass to
// clear them).
__global__ void clear_tickets_kernel(unsigned int *counters, int B) {
  pdl_wait();
  for (int b = threadIdx.x; b < B; b += blockDim.x) counters[b] = 0u;
}

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
  return SD_OK;
}

// Tokens per draw CTA: the race of one sequence is split so that all B sequences together give
// about one wave of CTAs; multiples of 1024 tokens.
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

// Clusters of each size (1, 2, 4, 8, 16 CTAs per sequence) the device holds at once for the
// decision kernel at one CTA per SM (looked up once per device; 0 where a size cannot run).
static const int *active_clusters(size_t smem) {
  static int cache[64][5];
  static bool done[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (done[dev]) return cache[dev];
  cudaFuncSetAttribute(accept_decide_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaFuncSetAttribute(accept_decide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem);
  for (int i = 0; i < 5; ++i) {
    const int cl = 1 << i;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cl, 1, 1);
    cfg.blockDim = dim3(kDecideThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, accept_decide_kernel, &cfg) != cudaSuccess) n = 0;
    cache[dev][i] = n;
  }
  cudaGetLastError();
  done[dev] = true;
  return cache[dev];
}

// Launch shape of the decision pass: cluster size (CTAs per sequence), tokens per CTA, bulk
// copies per row slice and the thread count.  As many CTAs per sequence as keep B x cluster
// within one CTA per SM (every CTA streams with a 3 x 64 KB ring), at least 1024 tokens each.
struct DecideShape {
  int cl, slice, npieces, threads;
  size_t smem;
};

static DecideShape decide_shape(int B, int V) {
  DecideShape s;
  const size_t full_smem = (size_t)kStages * kPiece * 4;
  // cluster size: fewest waves of clusters per CTA-slice of the vocabulary, i.e. the smallest
  // ceil(B / resident clusters) / cl; at least 1024 tokens per CTA
  const int *act = active_clusters(full_smem);
  int cl = 1;
  double best = -1.0;
  for (int i = 0; i < 5; ++i) {
    const int c = 1 << i;
    if (c > 1 && (V + c - 1) / c < 1024) break;
    const int n = act != nullptr ? act[i] : (c == 1 ? 1 : 0);
    if (n <= 0) continue;
    const double cost = (double)((B + n - 1) / n) / c;
    if (best < 0.0 || cost <= best) {
      best = cost;
      cl = c;
    }
  }
  s.cl = cl;
  int slice = (V + cl - 1) / cl;
  slice = (slice + 3) & ~3;
  s.slice = slice;
  s.npieces = (slice + kPiece - 1) / kPiece;
  const int piece = ((slice + s.npieces - 1) / s.npieces + 3) & ~3;
  // threads: enough for one float4 per thread of a piece, 32 .. kDecideThreads
  int th = (piece / 4 + 31) / 32 * 32;
  s.threads = th < 32 ? 32 : (th > kDecideThreads ? kDecideThreads : th);
  s.smem = (size_t)kStages * piece * 4;
  return s;
}

static size_t ws_size(const sd_accept_desc *d) {
  if (validate(d) != SD_OK) return 0;
  return round_up((size_t)d->batch * sizeof(Record), 256) +
         round_up((size_t)d->batch * ndraw_of(d->batch, d->vocab) * 48, 256) +
         round_up((size_t)d->batch * 4, 256);
}

}  // namespace acc
}  // namespace sdv

extern "C" {

size_t sd_accept_workspace_size(const sd_accept_desc *desc) { return sdv::acc::ws_size(desc); }

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
  p.rps = p.n_q + (sampling ? p.k : 0);
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
  uint8_t *w8 = reinterpret_cast<uint8_t *>(ws);
  p.rec = reinterpret_cast<Record *>(w8);
  w8 += round_up((size_t)p.B * sizeof(Record), 256);
  p.cand = reinterpret_cast<float4 *>(w8);
  w8 += round_up((size_t)p.B * p.ndraw * 48, 256);
  p.counters = reinterpret_cast<unsigned int *>(w8);
  p.status = device_status_word();
  cudaStream_t st = (cudaStream_t)stream;
  const bool plain = sampling && p.k == 0;
  if (plain) {
    if (launch(clear_tickets_kernel, dim3(1), dim3(kDrawThreads), 0, st, p.counters, p.B) !=
        cudaSuccess)
      return SD_ERR_CUDA;
  } else {
    const DecideShape ds = decide_shape(p.B, p.V);
    p.cl = ds.cl;
    p.slice = ds.slice;
    p.npieces = ds.npieces;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ds.cl * p.B, 1, 1);
    cfg.blockDim = dim3(ds.threads, 1, 1);
    cfg.dynamicSmemBytes = ds.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ds.cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, accept_decide_kernel, p) != cudaSuccess) return SD_ERR_CUDA;
    if (!sampling) return SD_OK;  // greedy: the decision pass wrote the outputs
  }
  return cuda_status(
      launch(accept_draw_kernel, dim3(p.B, p.ndraw), dim3(kDrawThreads), 0, st, p));
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

// Device address of the scratch array on the current device, looked up again whenever the
// current context is not the one of the cached address (e.g. after a device reset).  A symbol's
// host-side name is not a device address, so it is never passed to a kernel directly.
static void *noalloc_scratch() {
  static SymbolSlot slot;
  return symbol_address(slot, g_accept_noalloc_scratch);
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
  // The per-sequence tickets in the scratch are cleared at the start of every call (by the
  // decision kernel, or a one-block kernel for a plain draw), and every other byte the kernels
  // read is written earlier in the same call, so the array's leftover contents from an earlier
  // call do not matter.
  return sd_accept(desc, target_logits, draft_logits, draft_tokens, n_accepted, out_tokens,
                   margin_flags, scratch, (size_t)SD_ACCEPT_NOALLOC_MAX_SCRATCH, stream);
}
