// Commit of the accepted prefix and rollback of the rejected positions (sm_100a).
//
// "Gemma 4 MTP: drafter drafts, target verifies", section "basic structure of speculative
// decoding": only the prefix up to the rejected position is kept; Gemma 4 MTP serving guide,
// section 4: drafts after the first rejection are discarded.  The verify step wrote K/V for
// positions L .. L+k; L .. L+a are kept (new length L + a + 1), L+a+1 .. L+k are rolled back.
// The next hidden row of the drafter is the target's activation at the last kept position
// (first page, section "drafter internal architecture").
#include "common.cuh"
#include "host.cuh"

namespace sdv {
namespace cmt {

constexpr int kMaxPoison = 8;

struct PoisonList {
  void *cache[kMaxPoison];
  int h_kv[kMaxPoison];
  int head_dim[kMaxPoison];
  int is_bf16[kMaxPoison];
  int n;
};

struct Params {
  int B, k, n_q, bs, mbps, num_blocks, d, hidden_bytes, vec16;
  const int32_t *table;
  int32_t *ctx_len;
  const int32_t *n_acc;
  int32_t *slots;
  const uint8_t *hidden;
  uint8_t *next_hidden;
  PoisonList poison;
  unsigned long long *step_ptr;
  int *status;
};

__global__ void commit_kernel(const Params p) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x;
  __shared__ int s_a, s_L;
  if (threadIdx.x == 0) {
    int a = p.n_acc[b];
    const int L = p.ctx_len[b];
    if (a < 0 || a > p.k || L < 0) {
      record_status(p.status, SD_ERR_DEVICE);
      a = -1;
    }
    s_a = a;
    s_L = L;
  }
  __syncthreads();
  const int a = s_a, L = s_L;
  if (b == 0 && threadIdx.x == 0 && p.step_ptr != nullptr) *p.step_ptr += 1ull;
  if (a < 0) return;
  for (int j = threadIdx.x; j < p.n_q; j += blockDim.x) {
    int slot = -1;
    if (j <= a) {
      const int pos = L + j;
      const int bidx = pos / p.bs;
      const int blk = bidx < p.mbps ? p.table[(size_t)b * p.mbps + bidx] : -1;
      if (blk < 0 || blk >= p.num_blocks)
        record_status(p.status, SD_ERR_DEVICE);
      else
        slot = blk * p.bs + pos % p.bs;
    }
    p.slots[(size_t)b * p.n_q + j] = slot;
  }
  if (p.hidden != nullptr && p.next_hidden != nullptr) {
    const size_t row = (size_t)p.d * p.hidden_bytes;
    const uint8_t *src = p.hidden + ((size_t)b * p.n_q + a) * row;
    uint8_t *dst = p.next_hidden + (size_t)b * row;
    if (p.vec16) {  // 16-byte aligned rows: vector copy (the loads overlap)
      const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
      uint4 *d4 = reinterpret_cast<uint4 *>(dst);
      for (size_t i = threadIdx.x; i < row / 16; i += blockDim.x) d4[i] = s4[i];
    } else {
      for (size_t i = threadIdx.x; i < row; i += blockDim.x) dst[i] = src[i];
    }
  }
  for (int c = 0; c < p.poison.n; ++c) {
    const int H = p.poison.h_kv[c], D = p.poison.head_dim[c];
    for (int j = a + 1; j <= p.k; ++j) {
      const int pos = L + j;
      const int bidx = pos / p.bs;
      const int blk = bidx < p.mbps ? p.table[(size_t)b * p.mbps + bidx] : -1;
      if (blk < 0 || blk >= p.num_blocks) {
        if (threadIdx.x == 0) record_status(p.status, SD_ERR_DEVICE);
        continue;
      }
      for (int i = threadIdx.x; i < H * D; i += blockDim.x) {
        const int g = i / D, e = i % D;
        const size_t off = (((size_t)blk * H + g) * p.bs + pos % p.bs) * D + e;
        if (p.poison.is_bf16[c])
          reinterpret_cast<uint16_t *>(p.poison.cache[c])[off] = 0x7FC0u;  // bf16 NaN
        else
          reinterpret_cast<float *>(p.poison.cache[c])[off] = __int_as_float(0x7FC00000);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) p.ctx_len[b] = L + a + 1;
}

}  // namespace cmt
}  // namespace sdv

extern "C" sd_status sd_commit(const sd_commit_desc *desc, const int32_t *block_table,
                               int32_t *ctx_len, const int32_t *n_accepted,
                               int32_t *committed_slots, const void *hidden, void *next_hidden,
                               sd_stream stream) {
  using namespace sdv;
  using namespace sdv::cmt;
  if (!desc || !block_table || !ctx_len || !n_accepted || !committed_slots)
    return SD_ERR_INVALID_ARG;
  if (desc->batch < 1 || desc->k < 0 || desc->block_size < 1 || desc->max_blocks_per_seq < 1 ||
      desc->num_blocks < 1 || desc->n_poison < 0)
    return SD_ERR_INVALID_ARG;
  if ((hidden == nullptr) != (next_hidden == nullptr)) return SD_ERR_INVALID_ARG;
  if (hidden && (desc->d < 1 || (desc->hidden_dtype != SD_F32 && desc->hidden_dtype != SD_BF16)))
    return SD_ERR_INVALID_ARG;
  if (desc->n_poison > kMaxPoison) return SD_ERR_UNSUPPORTED;
  if (desc->n_poison > 0 && !desc->poison) return SD_ERR_INVALID_ARG;
  Params p{};
  p.B = desc->batch;
  p.k = desc->k;
  p.n_q = desc->k + 1;
  p.bs = desc->block_size;
  p.mbps = desc->max_blocks_per_seq;
  p.num_blocks = desc->num_blocks;
  p.d = desc->d;
  p.hidden_bytes = desc->hidden_dtype == SD_BF16 ? 2 : 4;
  p.table = block_table;
  p.ctx_len = ctx_len;
  p.n_acc = n_accepted;
  p.slots = committed_slots;
  p.hidden = reinterpret_cast<const uint8_t *>(hidden);
  p.next_hidden = reinterpret_cast<uint8_t *>(next_hidden);
  p.vec16 = hidden != nullptr && aligned16(hidden) && aligned16(next_hidden) &&
            ((size_t)p.d * p.hidden_bytes) % 16 == 0;
  p.poison.n = desc->n_poison;
  for (int i = 0; i < desc->n_poison; ++i) {
    const sd_poison_cache &c = desc->poison[i];
    if (!c.cache || c.h_kv < 1 || c.head_dim < 1 || (c.dtype != SD_F32 && c.dtype != SD_BF16))
      return SD_ERR_INVALID_ARG;
    p.poison.cache[i] = c.cache;
    p.poison.h_kv[i] = c.h_kv;
    p.poison.head_dim[i] = c.head_dim;
    p.poison.is_bf16[i] = c.dtype == SD_BF16;
  }
  p.step_ptr = reinterpret_cast<unsigned long long *>(desc->step_ptr);
  p.status = device_status_word();
  return cuda_status(launch(commit_kernel, dim3(p.B), dim3(256), 0, (cudaStream_t)stream, p));
}
