// contract.cuh -- the fixed constants of the reduction contract and the
// device error bits, shared by every kernel of the library.
//
// The KV context of a row is cut into splits of kSplitTokens tokens from
// absolute position 0 (the "KV chunk" of RL-Kernel PR #284 "feat(attention):
// add CP backward drift validation", Changes: fixed global_block_index merge
// order), each walked in tiles of kTileTokens tokens.  Neither constant
// depends on the batch, the SM count or the block size.
#pragma once

namespace pkv {

constexpr int kSplitTokens = 4096;
constexpr int kTileTokens = 128;

// Within a split, a row's running max m (base-2 units) rises to a tile's max
// only when that exceeds it by more than kMaxSlack; p = 2^(s - m) then stays
// below 2^kMaxSlack, and the P.V products, accumulated on the tensor cores
// over the split's tiles, are rescaled (by 2^(m - m'), in place) only then.
constexpr float kMaxSlack = 8.f;

// Number of splits that hold keys [0, n): ceil(n / kSplitTokens), 0 for n <= 0.
__host__ __device__ constexpr int splits_for(int n) {
  return n > 0 ? (n + kSplitTokens - 1) / kSplitTokens : 0;
}

// Device error bits (PKV_DEVERR_* in pagedkv.h).
constexpr int kErrBadBlock = 1;
constexpr int kErrTableWidth = 2;
constexpr int kErrTimeout = 4;
constexpr int kErrQueryLen = 8;
constexpr int kErrSeqLen = 16;

}  // namespace pkv
