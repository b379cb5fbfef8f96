// State copies between chunks: capsule snapshot / restore / fork of the prefix KV and x.
//
// FlashRT-PAI overview (mechanism 3, execution-state capsules) and the FlashRT walkthrough
// ("serving/": snapshot, restore, fork, time travel of the resident state) describe the
// operation: the state a graph replay depends on is copied out of and back into the named
// device buffers, optionally gathering samples.  Here that is one strided row copy: a row
// (one key or value vector, or one sample's action chunk) is moved by one warp with 16- or
// 4-byte words, rows indexed (outer, sample, mid, row) with independent byte strides on
// the two sides and a sample map on the source side.
#include "internal.h"

namespace fr {

namespace {

template <typename W>
__global__ void __launch_bounds__(256) k_state_copy(const __grid_constant__ RowCopy c) {
  const long long rows_per_part = c.n_outer * c.n_sample * c.n_mid * c.n_row;
  const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (r >= rows_per_part * c.parts) return;
  const int part = static_cast<int>(r / rows_per_part);
  long long q = r - part * rows_per_part;
  const long long p = q % c.n_row;
  q /= c.n_row;
  const long long m = q % c.n_mid;
  q /= c.n_mid;
  const int b = static_cast<int>(q % c.n_sample);
  const long long o = q / c.n_sample;
  const int bs = c.map[b];
  const W* src = reinterpret_cast<const W*>(c.src[part] + o * c.s_outer + bs * c.s_sample + m * c.s_mid + p * c.s_row);
  W* dst = reinterpret_cast<W*>(c.dst[part] + o * c.d_outer + b * c.d_sample + m * c.d_mid + p * c.d_row);
  for (int w = threadIdx.x & 31; w < c.row_words; w += 32) dst[w] = src[w];
}

bool aligned16(long long v) { return (v & 15) == 0; }

}  // namespace

void launch_state_copy(RowCopy c, cudaStream_t s) {
  // 16-byte words when every row start on both sides is 16-byte aligned, 4-byte words otherwise
  bool w16 = aligned16(c.row_bytes) && aligned16(c.s_outer) && aligned16(c.s_sample) && aligned16(c.s_mid) &&
             aligned16(c.s_row) && aligned16(c.d_outer) && aligned16(c.d_sample) && aligned16(c.d_mid) &&
             aligned16(c.d_row);
  for (int i = 0; i < c.parts; ++i)
    w16 = w16 && aligned16(reinterpret_cast<long long>(c.src[i])) && aligned16(reinterpret_cast<long long>(c.dst[i]));
  const long long rows = c.parts * c.n_outer * c.n_sample * c.n_mid * c.n_row;
  if (rows <= 0) return;
  const unsigned blocks = static_cast<unsigned>((rows + 7) / 8);
  if (w16) {
    c.row_words = static_cast<int>(c.row_bytes / 16);
    k_state_copy<uint4><<<blocks, 256, 0, s>>>(c);
  } else {
    c.row_words = static_cast<int>(c.row_bytes / 4);
    k_state_copy<uint32_t><<<blocks, 256, 0, s>>>(c);
  }
}

}  // namespace fr
