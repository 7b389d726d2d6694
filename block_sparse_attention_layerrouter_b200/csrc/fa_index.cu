// fa_index.cu -- CSR of the block-sparse pattern ("Flux Attention",
// implementation paragraph: 64-token blocks, sink tokens kept): row i lists,
// ascending and once each, the sink blocks j < sink_blocks (j <= i) and the
// window blocks max(0, i - win_blocks + 1) .. i.
//
// One CTA of 1024 threads: each thread counts a contiguous run of rows in
// closed form, a block-wide exclusive scan gives the row offsets, and each
// thread writes its rows.  The pattern is tiny (268,191 entries at 256K
// tokens with a 4096-token window), so one CTA is enough.
#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {
namespace index {

constexpr int NT = 1024;

FA_DEV void row_parts(int i, int sb, int wb, int &a, int &lo) {
  a = min(sb, i + 1);                 // sink blocks 0 .. a-1
  lo = max(a, i - wb + 1);            // window blocks lo .. i (after the sinks)
}

__global__ void __launch_bounds__(NT) csr_kernel(int nrows, int sb, int wb, int32_t *row_ptr,
                                                 int32_t *col_idx) {
  __shared__ long long sums[NT];
  const int t = threadIdx.x;
  const int per = (nrows + NT - 1) / NT;
  const int r0 = min(nrows, t * per), r1 = min(nrows, r0 + per);
  long long cnt = 0;
  for (int i = r0; i < r1; ++i) {
    int a, lo;
    row_parts(i, sb, wb, a, lo);
    cnt += a + (i - lo + 1);
  }
  sums[t] = cnt;
  __syncthreads();
  // Hillis-Steele inclusive scan over the per-thread counts.
  for (int off = 1; off < NT; off <<= 1) {
    const long long v = t >= off ? sums[t - off] : 0;
    __syncthreads();
    sums[t] += v;
    __syncthreads();
  }
  long long pos = sums[t] - cnt;
  for (int i = r0; i < r1; ++i) {
    int a, lo;
    row_parts(i, sb, wb, a, lo);
    row_ptr[i] = static_cast<int32_t>(pos);
    for (int j = 0; j < a; ++j) col_idx[pos++] = j;
    for (int j = lo; j <= i; ++j) col_idx[pos++] = j;
  }
  if (t == NT - 1) row_ptr[nrows] = static_cast<int32_t>(sums[NT - 1]);
}

}  // namespace index

long long index_nnz(int nrows, int sb, int wb) {
  long long n = 0;
  for (int i = 0; i < nrows; ++i) {
    const int a = sb < i + 1 ? sb : i + 1;
    const int w0 = i - wb + 1;
    const int lo = a > w0 ? a : w0;
    n += a + (i - lo + 1);
  }
  return n;
}

int launch_index(int nrows, int sb, int wb, int32_t *row_ptr, int32_t *col_idx,
                 cudaStream_t stream) {
  index::csr_kernel<<<1, index::NT, 0, stream>>>(nrows, sb, wb, row_ptr, col_idx);
  note_launch();
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace fa
