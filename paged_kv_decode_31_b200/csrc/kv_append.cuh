// kv_append.cuh -- write new K/V tokens into paged cache blocks.
//
// Token t of sequence b goes to position p = seqlens[b] - seq_bias + t: block
// block_table[b][p / block_size], slot p % block_size, addressed with the
// cache's real element strides.  The bf16 bits are copied unchanged with
// 128-bit loads and stores ([WS1] "KV-cache path consistency (prefill &
// decode)", Scope: the stored-KV dtype and layout must add no difference
// between the path that wrote the cache and the path that reads it).
#pragma once

#include <cstdint>

#include "packed.cuh"

namespace pkv {

struct AppendParams {
  const uint16_t *k_new, *v_new;
  int64_t kn_sb, kn_st, kn_sh, vn_sb, vn_st, vn_sh;
  uint16_t *k_cache, *v_cache;
  int64_t k_sb, k_ss, k_sh, v_sb, v_ss, v_sh;
  int64_t num_blocks;
  const int32_t *block_table;
  int64_t bt_stride;
  int max_blocks_per_seq;
  const int32_t *seqlens;
  int batch, n_new, Hkv, chunks;  // chunks = D / 8 (16-byte pieces per head row)
  int block_shift;
  // 0 for pkv_kv_append (seqlens before the append); n_new when the attention
  // call appends (seqlens after it): then positions below 0 are skipped
  // without an error, as the fused path does.
  int seq_bias;
  // Packed new tokens (cu_new != null): k_new / v_new are [total_new, Hkv, D]
  // (token stride kn_st / vn_st) and token tf belongs to sequence
  // b = seq_of_token(cu_new, batch, tf) at t = tf - cu_new[b].
  const int32_t *cu_new;
  int total_new;
  int32_t *err;
};

// One block per new token (blockIdx.x: b * n_new + t, or the packed index):
// one thread resolves the token's sequence, cache position and block once,
// then the block's threads copy its Hkv x (D / 8) 16-byte pieces.
__global__ void __launch_bounds__(256) kv_append_kernel(const __grid_constant__ AppendParams p) {
  __shared__ int64_t s_dst_k, s_dst_v, s_src_k, s_src_v;  // element offsets (-1: skip the token)
  const int64_t r = blockIdx.x;
  if (threadIdx.x == 0) {
    int b, t;
    int64_t kn_off, vn_off;
    if (p.cu_new) {
      b = seq_of_token(p.cu_new, p.batch, r);
      t = static_cast<int>(r - __ldg(p.cu_new + b));
      kn_off = r * p.kn_st;
      vn_off = r * p.vn_st;
    } else {
      t = static_cast<int>(r % p.n_new);
      b = static_cast<int>(r / p.n_new);
      kn_off = b * p.kn_sb + t * p.kn_st;
      vn_off = b * p.vn_sb + t * p.vn_st;
    }
    int64_t dk = -1, dv = -1;
    const int64_t pos = static_cast<int64_t>(__ldg(p.seqlens + b)) - p.seq_bias + t;
    const int64_t bi = pos >> p.block_shift;
    if (pos < 0 && p.seq_bias > 0) {
      // before the sequence's start in the fused path: nothing to write
    } else if (pos < 0 || bi >= p.max_blocks_per_seq) {
      if (p.err) atomicOr(p.err, 2);
    } else {
      const int32_t blk = __ldg(p.block_table + b * p.bt_stride + bi);
      if (blk < 0 || static_cast<int64_t>(blk) >= p.num_blocks) {
        if (p.err) atomicOr(p.err, 1);
      } else {
        const int64_t slot = pos & ((int64_t{1} << p.block_shift) - 1);
        dk = blk * p.k_sb + slot * p.k_ss;
        dv = blk * p.v_sb + slot * p.v_ss;
      }
    }
    s_dst_k = dk;
    s_dst_v = dv;
    s_src_k = kn_off;
    s_src_v = vn_off;
  }
  __syncthreads();
  const int64_t dk = s_dst_k, dv = s_dst_v;
  if (dk < 0) return;  // uniform over the block
  const uint16_t *kn = p.k_new + s_src_k, *vn = p.v_new + s_src_v;
  const int n = p.Hkv * p.chunks;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int h = i / p.chunks, c = i - h * p.chunks;
    const uint4 kv = __ldg(reinterpret_cast<const uint4 *>(kn + h * p.kn_sh) + c);
    const uint4 vv = __ldg(reinterpret_cast<const uint4 *>(vn + h * p.vn_sh) + c);
    reinterpret_cast<uint4 *>(p.k_cache + dk + h * p.k_sh)[c] = kv;
    reinterpret_cast<uint4 *>(p.v_cache + dv + h * p.v_sh)[c] = vv;
  }
}

}  // namespace pkv
