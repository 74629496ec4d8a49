// Lossless acceptance of k drafts, correction / bonus draw, greedy rule (sm_100a).
//
// The rule (pages cite Leviathan et al. for it: Google blog translation, section "how
// speculative decoding works"; property stated in "Gemma 4 MTP: drafter drafts, target
// verifies", section "basic structure of speculative decoding"): accept d_i iff
// u_i < p_i(d_i) / q_i(d_i); at the first rejection emit x ~ norm(max(0, p_i - q_i)); if all
// are accepted emit the bonus x ~ p_{k+1}.  T = 0: accept iff d_i == argmax, emit argmax.
//
// Two kernels at T > 0 (a plain draw, k = 0, runs a ticket clear and the second), two at T = 0
// (the first and accept_decide):
//  1. accept_stats: one CTA per (logit row, token chunk) over every row the sequences need (the
//     k+1 target rows and, for T > 0, the k draft rows), sized to one wave of CTAs: online max /
//     sum of exp(x / T) of the chunk (T > 0), or its top two values and the argmax (T = 0),
//     with 16-byte loads kept in flight.  It also clears the draw's tickets.
//  The decisions (decide_seq): a CTA merges the chunks of each row of its sequence (a warp per
//     row, fixed order) and tests the k drafts lane-parallel: the accepted count, the
//     acceptance margin flag and the normalisers of the draw row.  At T = 0 accept_decide (one
//     CTA per sequence) takes them and writes the outputs; at T > 0 every CTA of accept_mass
//     takes them first (all reach the same ones), which saves a launch between the passes.
//  2. accept_mass: the categorical draw as a two-level exponential race.  CTAs per (sequence,
//     run of 512-token groups), one wave of them, reduce each group of the draw row to its mass
//     (max(0, p - q) after a rejection; p for the bonus draw and plain draws) with the sums the
//     margin bounds need.  The last CTA of a sequence (atomic ticket; no waiting) races the
//     groups, key_g = log2 W_g - log2(-ln(1 - V_g)) with the group's Philox uniform, then the
//     winning group's 512 tokens, key_v = log2 w_v - log2(-ln(1 - V_v)), keeping at each level
//     the winner's lowest possible key and the highest possible key of every other competitor
//     under the float32 error model of the margin rule, and writes the outputs.  The generator
//     runs for the groups and one group's tokens instead of every token of the row.
#include <cfloat>

#include "common.cuh"
#include "host.cuh"
#include "philox.cuh"

namespace sdv {
namespace acc {

constexpr int kStatThreads = 256;
constexpr int kChunk = 8192;        // tokens per statistics CTA at least
constexpr int kDecideThreads = 256;  // the decisions also run inside the group-mass CTAs
constexpr int kMaxRows = 31;        // rows per sequence: 2k + 1 with k <= 15
constexpr int kMassSlots = 592;     // group-mass CTAs aimed at: one wave at 4 CTAs per SM
constexpr int kMassThreads = 256;   // the last CTA races 2 groups / 2 tokens per thread
constexpr int kGroup = 512;         // tokens per group of the two-level race
constexpr uint32_t kGroupPurpose = 16;  // group uniforms: the draw's purpose + 16
constexpr float kMargin = 1e-4f;    // spec margin on |u - p/q|; also for draws, argmaxes
constexpr float kRelP = 1e-5f;      // float32 error bound assumed on a probability p_v or q_v
constexpr float kAbsKey = 1e-5f;    // float32 error bound assumed on ln E_v and z_v / T
constexpr float kLog2e = 1.4426950408889634f;
// the race keys are kept in log2 units: the natural-log margin and bounds scaled by log2(e)
constexpr float kMargin2 = kMargin * kLog2e;
constexpr float kAbsKey2 = kAbsKey * kLog2e;

// Decision record of one sequence (T > 0), taken by each CTA of the draw.
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
  int rps;           // rows per sequence read by the statistics pass
  int nchunks, stats_chunk;
  int ngroups;       // token groups of a row, ceil(V / kGroup)
  int nmass, mass_groups;  // group-mass CTAs per sequence, groups per CTA
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
  float4 *stats;           // [B * rps][nchunks] chunk partials
  float4 *gm;              // [B][ngroups] group masses of the draw row
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

__device__ __forceinline__ bool race_flag(const Race &r) { return r.hi2 > r.lo1 - kMargin2; }

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

// ------------------------------------------------------------------ statistics kernel

__global__ void __launch_bounds__(kStatThreads) accept_stats_kernel(const Params p) {
  pdl_wait();  // many waves: no early trigger, so the next kernel does not take their slots
  const int rr = blockIdx.x, c = blockIdx.y;
  const int b = rr / p.rps, ri = rr - b * p.rps;
  // the tickets of the group-mass kernel that follows start from zero
  if (p.T > 0.f && ri == 0 && c == 0 && threadIdx.x == 0) p.counters[b] = 0u;
  const float *row = seq_row(p, b, ri);
  const int v0 = c * p.stats_chunk;
  const int v1 = min(p.V, v0 + p.stats_chunk);
  const float4 *row4 = reinterpret_cast<const float4 *>(row + v0);
  const int n4 = max(0, v1 - v0) >> 2;
  __shared__ float4 red[kStatThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (p.T > 0.f) {
    // a batch of PER independent loads per thread, then their max, then the sum, merged
    // online across batches
    constexpr int PER = 8;
    const float inv_t = 1.f / p.T;
    float m = -INFINITY, s = 0.f;
    for (int base = 0; base < n4; base += PER * kStatThreads) {
      float4 x[PER];
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        const int i = base + threadIdx.x + u * kStatThreads;
        x[u] = i < n4 ? __ldg(row4 + i)
                      : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      }
      if (p.T != 1.f) {
#pragma unroll
        for (int u = 0; u < PER; ++u)
          x[u] = make_float4(x[u].x * inv_t, x[u].y * inv_t, x[u].z * inv_t, x[u].w * inv_t);
      }
      float mb = -INFINITY, sb = 0.f;
#pragma unroll
      for (int u = 0; u < PER; ++u)
        mb = fmaxf(mb, fmaxf(fmaxf(x[u].x, x[u].y), fmaxf(x[u].z, x[u].w)));
      if (mb != -INFINITY) {
        const float ml = mb * kLog2e;
#pragma unroll
        for (int u = 0; u < PER; ++u)
          sb += (exp2f(fmaf(x[u].x, kLog2e, -ml)) + exp2f(fmaf(x[u].y, kLog2e, -ml))) +
                (exp2f(fmaf(x[u].z, kLog2e, -ml)) + exp2f(fmaf(x[u].w, kLog2e, -ml)));
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
      for (int w = 1; w < kStatThreads / 32; ++w) ms_merge(M, S, red[w].x, red[w].y);
      p.stats[(size_t)rr * p.nchunks + c] = make_float4(M, S, 0.f, 0.f);
    }
  } else {
    Top2 cd{-INFINITY, -INFINITY, -1};
    for (int i = threadIdx.x; i < n4; i += kStatThreads) {
      const float4 x4 = __ldg(row4 + i);
      const int v = v0 + 4 * i;
      top2_push(cd, x4.x, v);
      top2_push(cd, x4.y, v + 1);
      top2_push(cd, x4.z, v + 2);
      top2_push(cd, x4.w, v + 3);
    }
    for (int off = 16; off > 0; off >>= 1) cd = top2_merge(cd, top2_shfl(cd, off));
    if (lane == 0) red[warp] = make_float4(cd.g1, __int_as_float(cd.v1), cd.g2, 0.f);
    __syncthreads();
    if (threadIdx.x == 0) {
      Top2 t{red[0].x, red[0].z, __float_as_int(red[0].y)};
      for (int w = 1; w < kStatThreads / 32; ++w)
        t = top2_merge(t, Top2{red[w].x, red[w].z, __float_as_int(red[w].y)});
      p.stats[(size_t)rr * p.nchunks + c] = make_float4(t.g1, __int_as_float(t.v1), t.g2, 0.f);
    }
  }
}

// ------------------------------------------------------------------ decisions

// The decisions of sequence b, taken by one CTA of kDecideThreads threads from the merged row
// statistics: greedy (T = 0) writes the outputs; sampling leaves the record of the draw in
// *rec_out (shared memory; valid after the CTA's next barrier, which every thread must reach).
__device__ __forceinline__ void decide_seq(const Params &p, int b, float4 *s_row,
                                           uint32_t *s_step, Record *rec_out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool sampling = p.T > 0.f;
  if (threadIdx.x == 0) *s_step = counter_step(p);
  // the drafts and their logits, loaded before the merge so that their round trips overlap it
  // (warp 0, lane i - 1 for draft i)
  int d = -1;
  float zd = 0.f, yd = 0.f;
  if (warp == 0 && lane < p.k) {
    d = p.drafts[(size_t)b * p.k + lane];
    if (sampling && d >= 0 && d < p.V) {
      zd = p.z[(size_t)(b * p.n_q + lane) * p.ld_t + d];
      yd = p.y[((size_t)b * p.k + lane) * p.ld_d + d];
    }
  }
  // merge the chunks of each row (one warp per row, lanes over chunks, fixed order)
  for (int ri = warp; ri < p.rps; ri += kDecideThreads / 32) {
    const float4 *st = p.stats + (size_t)(b * p.rps + ri) * p.nchunks;
    float4 v;
    if (sampling) {
      float M = -INFINITY, S = 0.f;
      for (int c = lane; c < p.nchunks; c += 32) ms_merge(M, S, st[c].x, st[c].y);
      for (int off = 16; off > 0; off >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, M, off);
        const float s2 = __shfl_xor_sync(0xffffffffu, S, off);
        ms_merge(M, S, m2, s2);
      }
      v = make_float4(M, S, 0.f, 0.f);
    } else {
      Top2 t{-INFINITY, -INFINITY, -1};
      for (int c = lane; c < p.nchunks; c += 32)
        t = top2_merge(t, Top2{st[c].x, st[c].z, __float_as_int(st[c].y)});
      for (int off = 16; off > 0; off >>= 1) t = top2_merge(t, top2_shfl(t, off));
      v = make_float4(t.g1, __int_as_float(t.v1), t.g2, 0.f);
    }
    if (lane == 0) s_row[ri] = v;
  }
  __syncthreads();
  if (warp != 0) return;

  // ---- decisions (one warp): lane i-1 tests draft i; the first rejection stops the scan
  const uint32_t step = *s_step;
  const float inv_t = sampling ? 1.f / p.T : 1.f;
  bool acc = true;
  int flag = 0;
  if (lane < p.k) {
    const int rt = b * p.n_q + lane;
    const float4 sz = s_row[lane];
    if (d < 0 || d >= p.V) {
      record_status(p.status, SD_ERR_DEVICE);
      acc = false;
    } else if (sampling) {
      const float4 sy = s_row[p.n_q + lane];
      const float pd = expf(zd * inv_t - sz.x) / sz.y;
      const float qd = expf(yd * inv_t - sy.x) / sy.y;
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
  *rec_out = r;
}

static_assert(kDecideThreads == kMassThreads, "the group-mass CTAs take the decisions too");

// Greedy acceptance (T = 0): one CTA per sequence takes the decisions and writes the outputs.
__global__ void __launch_bounds__(kDecideThreads) accept_decide_kernel(const Params p) {
  __shared__ float4 s_row[kMaxRows];  // merged rows
  __shared__ uint32_t s_step;
  __shared__ Record s_rec;
  pdl_wait();
  decide_seq(p, blockIdx.x, s_row, &s_step, &s_rec);
}

// ------------------------------------------------------------------ group masses and the race

// Level-2 token of the race (log2 units):
//   draw from p (resid == false): key = zt log2(e) - lg2 E, bounds key -/+ 1e-5 (1 + |zt|)
//   residual (resid == true): key = lg2 w - lg2 E (w = max(0, p - q) > 0), its lower bound from
//   w - s and the upper bound of every token from w + s, s = 1e-5 (p + q), each -/+ 1e-5.
__device__ __forceinline__ void race_token(bool resid, float zt, float w, float sl, float lgE,
                                           int v, Race &cr) {
  if (!resid) {
    if (zt == -INFINITY) return;
    const float g = fmaf(zt, kLog2e, -lgE);
    const float err = kAbsKey2 * (1.f + fabsf(zt));
    race_push(cr, g, g - err, g + err, v);
    return;
  }
  if (w + sl > 0.f) {
    const float hi = __log2f(w + sl) - lgE + kAbsKey2;
    const float g = w > 0.f ? __log2f(w) - lgE : -INFINITY;
    if (g > cr.g1) {
      const float wl = w - sl;
      race_push(cr, g, wl > 0.f ? __log2f(wl) - lgE - kAbsKey2 : -INFINITY, hi, v);
    } else {
      cr.hi2 = fmaxf(cr.hi2, hi);
    }
  }
}

// Reduces a race over the CTA (lowest index first on equal keys); every thread gets the result.
__device__ __forceinline__ Race race_block(Race r, Race *s_red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int off = 16; off > 0; off >>= 1) {
    const Race o = race_shfl(r, off);
    r = (lane & off) ? race_merge(o, r) : race_merge(r, o);
  }
  __syncthreads();  // s_red may still be read from an earlier reduction
  if (lane == 0) s_red[warp] = r;
  __syncthreads();
  Race t = s_red[0];
  for (int w = 1; w < kMassThreads / 32; ++w) t = race_merge(t, s_red[w]);
  return t;
}

// One CTA per (sequence, run of token groups).  Each warp reduces whole 512-token groups of the
// draw row (16 tokens a lane, 16-byte loads issued together):
//   draw from p:   (m_g, s_g, A_g) = group max of z / T, sum of exp(z / T - m_g), max |z / T|
//   residual:      (W_g, S_g, P_g) = sums of max(0, p - q), of 1e-5 (p + q), and of p
// The last CTA of the sequence (atomic ticket, no waiting) races the groups (level 1, group
// uniforms), then the 512 tokens of the winning group (level 2, token uniforms), and writes the
// outputs.  An empty residual falls back to the race over p (flagged).
__global__ void __launch_bounds__(kMassThreads) accept_mass_kernel(const Params p) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x, c = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __shared__ Race s_red[kMassThreads / 32];
  __shared__ int s_last;
  __shared__ float4 s_row[kMaxRows];
  __shared__ uint32_t s_step;
  __shared__ Record s_rec;

  // Every CTA of the sequence takes the decisions itself (the same ones: they read the same
  // statistics), then reads the row they select.
  Record rec;
  if (p.k == 0) {  // plain draw: no decisions, unnormalised keys
    rec = Record{0, 0, 0u, 0, 0.f, 1.f, 0.f, 1.f};
  } else {
    decide_seq(p, b, s_row, &s_step, &s_rec);
    __syncthreads();
    rec = s_rec;
  }
  const int a = rec.a;
  const bool resid = a < p.k;
  const int rt = b * p.n_q + a;
  const float *zr = p.z + (size_t)rt * p.ld_t;
  const float *yr = resid ? p.y + ((size_t)b * p.k + a) * p.ld_d : nullptr;
  const bool unit_t = p.T == 1.f;
  const float inv_t = 1.f / p.T;
  const float isz = rec.isz, isy = rec.isy;
  const float mzl = rec.mz * kLog2e, myl = rec.my * kLog2e;
  float4 *gm = p.gm + (size_t)b * p.ngroups;

  const int g_end = min(p.ngroups, (c + 1) * p.mass_groups);
  for (int g = c * p.mass_groups + warp; g < g_end; g += kMassThreads / 32) {
    const int v0 = g * kGroup;
    const int n4 = min(kGroup, p.V - v0) >> 2;
    const float4 *z4 = reinterpret_cast<const float4 *>(zr + v0);
    const float4 *y4 = resid ? reinterpret_cast<const float4 *>(yr + v0) : nullptr;
    float4 zz[4], yy[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = lane + 32 * u;
      zz[u] = i < n4 ? __ldg(z4 + i) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      yy[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (resid && i < n4) yy[u] = __ldg(y4 + i);
    }
    float4 out;
    if (!resid) {
      float m = -INFINITY, A = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float *x = reinterpret_cast<float *>(&zz[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (!unit_t) x[e] *= inv_t;
          m = fmaxf(m, x[e]);
          if (x[e] != -INFINITY) A = fmaxf(A, fabsf(x[e]));
        }
      }
      for (int off = 16; off > 0; off >>= 1) {
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        A = fmaxf(A, __shfl_xor_sync(0xffffffffu, A, off));
      }
      float s = 0.f;
      if (m != -INFINITY) {
        const float ml = m * kLog2e;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float *x = reinterpret_cast<const float *>(&zz[u]);
#pragma unroll
          for (int e = 0; e < 4; ++e) s += ex2_approx(fmaf(x[e], kLog2e, -ml));
        }
      }
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      out = make_float4(m, s, A, 0.f);
    } else {
      float W = 0.f, S = 0.f, P = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (lane + 32 * u >= n4) continue;  // past the row's end
        const float *zx = reinterpret_cast<const float *>(&zz[u]);
        const float *yx = reinterpret_cast<const float *>(&yy[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float zt = unit_t ? zx[e] : zx[e] * inv_t;
          const float yt = unit_t ? yx[e] : yx[e] * inv_t;
          const float pv = ex2_approx(fmaf(zt, kLog2e, -mzl)) * isz;
          const float qv = ex2_approx(fmaf(yt, kLog2e, -myl)) * isy;
          W += fmaxf(pv - qv, 0.f);
          S += kRelP * (pv + qv);
          P += pv;
        }
      }
      for (int off = 16; off > 0; off >>= 1) {
        W += __shfl_xor_sync(0xffffffffu, W, off);
        S += __shfl_xor_sync(0xffffffffu, S, off);
        P += __shfl_xor_sync(0xffffffffu, P, off);
      }
      out = make_float4(W, S, P, 0.f);
    }
    if (lane == 0) gm[g] = out;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned int ticket = atomicAdd(&p.counters[b], 1u);
    s_last = ticket == (unsigned int)(p.nmass - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- last CTA of the sequence.  Level 1: the groups (thread t takes the group pair
  // 2t, 2t + 1: one Philox call)
  const uint32_t step = p.k == 0 ? counter_step(p) : rec.step;
  const uint32_t gpurpose = (uint32_t)p.purpose + kGroupPurpose;
  Race cr = race_empty();
  Race pb = race_empty();  // residual fallback: the race over the groups' p mass, g1 / v1 only
  for (int gp = threadIdx.x; 2 * gp < p.ngroups; gp += kMassThreads) {
    float U[2];
    token_uniform_pair(p.seed, step, (uint32_t)rt, gpurpose, (uint32_t)gp, U[0], U[1]);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int g = 2 * gp + e;
      if (g >= p.ngroups) break;
      const float4 q = __ldcg(gm + g);
      const float lgE = __log2f(neg_log1m(U[e]));
      if (!resid) {
        if (q.x == -INFINITY || !(q.y > 0.f)) continue;
        const float key = __log2f(q.y) + q.x * kLog2e - lgE;
        const float err = kAbsKey2 * (1.f + q.z);
        race_push(cr, key, key - err, key + err, g);
      } else {
        if (q.z > 0.f) {
          const float kp = __log2f(q.z) - lgE;
          if (kp > pb.g1) {
            pb.g1 = kp;
            pb.v1 = g;
          }
        }
        if (q.x + q.y > 0.f) {
          const float hi = __log2f(q.x + q.y) - lgE + kAbsKey2;
          const float key = q.x > 0.f ? __log2f(q.x) - lgE : -INFINITY;
          if (key > cr.g1) {
            const float wl = q.x - q.y;
            race_push(cr, key, wl > 0.f ? __log2f(wl) - lgE - kAbsKey2 : -INFINITY, hi, g);
          } else {
            cr.hi2 = fmaxf(cr.hi2, hi);
          }
        }
      }
    }
  }
  cr = race_block(cr, s_red);
  if (resid) pb = race_block(pb, s_red);
  // the residual race unless every residual weight came out 0: then the race over p, flagged
  // (a residual too small for float32 may still be positive)
  const bool empty = resid && cr.v1 < 0;
  int flag = rec.flag;
  if (empty || race_flag(cr)) flag = 1;
  int gsel = empty ? pb.v1 : cr.v1;
  if (gsel < 0) {  // no positive weight in the row at all
    gsel = 0;
    flag = 1;
  }
  const bool tok_resid = resid && !empty;

  // ---- level 2: the tokens of group gsel (thread t takes tokens 2t, 2t + 1)
  Race tr = race_empty();
  {
    const int v = gsel * kGroup + 2 * threadIdx.x;
    if (v < p.V) {  // V is a multiple of 4: both tokens exist
      float U[2];
      token_uniform_pair(p.seed, step, (uint32_t)rt, (uint32_t)p.purpose, (uint32_t)(v >> 1),
                         U[0], U[1]);
      const float2 z2 = __ldg(reinterpret_cast<const float2 *>(zr + v));
      const float2 y2 = tok_resid ? __ldg(reinterpret_cast<const float2 *>(yr + v))
                                  : make_float2(0.f, 0.f);
      const float zz[2] = {z2.x, z2.y}, yy[2] = {y2.x, y2.y};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float zt = unit_t ? zz[e] : zz[e] * inv_t;
        float w = 0.f, sl = 0.f;
        if (tok_resid) {
          const float yt = unit_t ? yy[e] : yy[e] * inv_t;
          const float pv = ex2_approx(fmaf(zt, kLog2e, -mzl)) * isz;
          const float qv = ex2_approx(fmaf(yt, kLog2e, -myl)) * isy;
          w = fmaxf(pv - qv, 0.f);
          sl = kRelP * (pv + qv);
        }
        const float lgE = __log2f(neg_log1m(U[e]));  // E == 0 gives -inf: that token wins
        race_token(tok_resid, zt, w, sl, lgE, v + e, tr);
      }
    }
  }
  tr = race_block(tr, s_red);
  if (threadIdx.x != 0) return;
  if (race_flag(tr)) flag = 1;
  int x = tr.v1;
  if (x < 0) {
    x = gsel * kGroup;
    flag = 1;
  }
  int32_t *o = p.out + (size_t)b * p.ld_o;
  for (int j = 0; j < p.n_q; ++j)
    o[j] = j < a ? p.drafts[(size_t)b * p.k + j] : (j == a ? x : -1);
  p.n_acc[b] = a;
  if (p.margin) p.margin[b] = flag;
  p.counters[b] = 0u;
}

// Zeroes the per-sequence tickets of the draw (plain draws, which have no statistics pass to
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

// Token groups per group-mass CTA: the groups of one sequence are split so that all B sequences
// together give about one wave of CTAs, at least one group per warp.
static int ngroups_of(int V) { return (V + kGroup - 1) / kGroup; }
static int mass_groups_of(int B, int V) {
  int per_seq = kMassSlots / (B > 0 ? B : 1);
  if (per_seq < 1) per_seq = 1;
  const int ng = ngroups_of(V);
  int m = (ng + per_seq - 1) / per_seq;
  constexpr int W = kMassThreads / 32;
  m = (m + W - 1) / W * W;
  return m;
}
static int nmass_of(int B, int V) {
  const int m = mass_groups_of(B, V);
  return (ngroups_of(V) + m - 1) / m;
}

static int nchunks_of(int V) { return (V + kChunk - 1) / kChunk; }

// Tokens per CTA of the statistics pass: kChunk, or more (multiples of 1024) when the rows
// times kChunk-token chunks would not fit in one wave of CTAs.  Never more chunks per row than
// nchunks_of(V), which sizes the workspace.
static int stats_chunk_of(int rows, int V) {
  static int occ_cache[64];
  int dev = 0;
  cudaGetDevice(&dev);
  int occ = dev >= 0 && dev < 64 ? occ_cache[dev] : 0;
  if (occ <= 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, accept_stats_kernel, kStatThreads,
                                                      0) != cudaSuccess ||
        occ <= 0)
      occ = 1;
    if (dev >= 0 && dev < 64) occ_cache[dev] = occ;
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

static size_t ws_size(const sd_accept_desc *d) {
  if (validate(d) != SD_OK) return 0;
  const size_t rows = (size_t)d->batch * (2 * d->k + 1);
  return round_up(rows * nchunks_of(d->vocab) * 16, 256) +
         round_up((size_t)d->batch * ngroups_of(d->vocab) * 16, 256) +
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
  p.ngroups = ngroups_of(desc->vocab);
  p.mass_groups = mass_groups_of(desc->batch, desc->vocab);
  p.nmass = nmass_of(desc->batch, desc->vocab);
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
  p.stats = reinterpret_cast<float4 *>(w8);
  w8 += round_up((size_t)p.B * (2 * p.k + 1) * nchunks_of(p.V) * 16, 256);
  p.gm = reinterpret_cast<float4 *>(w8);
  w8 += round_up((size_t)p.B * p.ngroups * 16, 256);
  p.counters = reinterpret_cast<unsigned int *>(w8);
  p.status = device_status_word();
  cudaStream_t st = (cudaStream_t)stream;
  const bool plain = sampling && p.k == 0;
  if (plain) {
    if (launch(clear_tickets_kernel, dim3(1), dim3(kMassThreads), 0, st, p.counters, p.B) !=
        cudaSuccess)
      return SD_ERR_CUDA;
  } else {
    p.stats_chunk = stats_chunk_of(p.B * p.rps, p.V);
    p.nchunks = (p.V + p.stats_chunk - 1) / p.stats_chunk;
    if (launch(accept_stats_kernel, dim3(p.B * p.rps, p.nchunks), dim3(kStatThreads), 0, st,
               p) != cudaSuccess)
      return SD_ERR_CUDA;
    if (!sampling)  // greedy: the decision pass writes the outputs
      return cuda_status(
          launch(accept_decide_kernel, dim3(p.B), dim3(kDecideThreads), 0, st, p));
  }
  return cuda_status(
      launch(accept_mass_kernel, dim3(p.B, p.nmass), dim3(kMassThreads), 0, st, p));
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
  // statistics kernel, or a one-block kernel for a plain draw), and every other byte the kernels
  // read is written earlier in the same call, so the array's leftover contents from an earlier
  // call do not matter.
  return sd_accept(desc, target_logits, draft_logits, draft_tokens, n_accepted, out_tokens,
                   margin_flags, scratch, (size_t)SD_ACCEPT_NOALLOC_MAX_SCRATCH, stream);
}
