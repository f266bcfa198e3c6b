// seq_table.cuh - sequence bookkeeping passed to kernels by value.
//
// Dense problems: every sequence has `len` tokens, padded to `pad_len`
// (a multiple of 128).  Varlen problems: packed sequences with host-side prefix
// sums copied into the kernel parameters (no device allocation needed).
#pragma once

#include <cstdint>

namespace sage {

constexpr int kMaxSeq = 1024;  // sequences per varlen call

struct SeqDense {
  int nseq;     // B
  int len;      // tokens per sequence
  int pad_len;  // len rounded up to 128
  int t_pad;    // nseq * pad_len
};

struct SeqVarlen {
  int nseq;
  int t_pad;
  int32_t cu[kMaxSeq + 1];    // packed token offset of each sequence
  int32_t poff[kMaxSeq + 1];  // padded token offset of each sequence
  int32_t cta[kMaxSeq + 1];   // first attention CTA of each sequence
};

// Where a sequence lives: its index, length, padded offset, and the element
// offset of its token 0 in an input tensor with strides (sb, st).
struct SeqPos {
  int b;
  int n;
  int off;
  int64_t base;
};

__host__ __device__ inline int seq_len(const SeqDense& s, int) { return s.len; }
__host__ __device__ inline int seq_len(const SeqVarlen& s, int b) { return s.cu[b + 1] - s.cu[b]; }
__host__ __device__ inline int seq_off(const SeqDense& s, int b) { return b * s.pad_len; }
__host__ __device__ inline int seq_off(const SeqVarlen& s, int b) { return s.poff[b]; }
__host__ __device__ inline int64_t seq_base(const SeqDense&, int b, int64_t sb, int64_t) {
  return static_cast<int64_t>(b) * sb;
}
__host__ __device__ inline int64_t seq_base(const SeqVarlen& s, int b, int64_t, int64_t st) {
  return static_cast<int64_t>(s.cu[b]) * st;
}

// Sequence containing padded token index tp (0 <= tp < t_pad).
__device__ inline int seq_of_padded(const SeqDense& s, int tp) { return tp / s.pad_len; }
__device__ inline int seq_of_padded(const SeqVarlen& s, int tp) {
  int lo = 0, hi = s.nseq - 1;  // largest b with poff[b] <= tp and a non-empty range
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.poff[mid] <= tp) lo = mid; else hi = mid - 1;
  }
  while (lo + 1 < s.nseq && s.poff[lo + 1] <= tp) ++lo;  // skip empty sequences
  return lo;
}

template <class Seq>
__device__ inline SeqPos locate(const Seq& s, int tp, int64_t sb, int64_t st) {
  SeqPos p;
  p.b = seq_of_padded(s, tp);
  p.n = seq_len(s, p.b);
  p.off = seq_off(s, p.b);
  p.base = seq_base(s, p.b, sb, st);
  return p;
}

}  // namespace sage
