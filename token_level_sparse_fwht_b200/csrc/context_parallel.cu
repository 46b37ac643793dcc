// Context-parallel decode: the merge of the ranks' softmax partials.
//
// A context of L_total positions is split into contiguous slices, one per rank
// (one GPU).  Each rank runs the fused decode kernel twice on its slice: phase 1
// exports the per-head cumulative histogram of Manhattan distances (no HBM array of
// distances or scores is written), the ranks all-gather the histograms, and phase 2
// resolves the global k-th distance and tie share by adding, at the few bins its
// two-level search reads, the other ranks' counts (and the lower ranks' for the tie
// share) to its own -- exactly as the CTAs of one cluster combine theirs -- then
// selects its part, attends over it and exports one softmax partial per head.  The
// ranks all-gather the partials and launch_cp_combine merges them.  The selection
// is the global top-k under (distance, position) with ties to the lower position,
// because a lower rank holds lower positions.
//
// Method: "Adamas: Hadamard Sparse Attention for Efficient Long-Context Inference",
// v2 abstract (distance-based top-k over compact codes, gather of the original KV
// states); the split over GPUs is this implementation's, the pages run one device.
#include "adamas_internal.cuh"

namespace adamas {

// One warp per (batch, query head) row; lane l owns coordinates 4l .. 4l+3.
// partials [world][rows][kPartStride] as the decode kernel exports them (m in the
// log2 domain, l, 0, 0, acc[128]); a partial with l = 0 is empty.  The world's
// (m, l) pairs are read by as many lanes at once and max-reduced across the warp,
// then every lane has its world 16-byte accumulator loads in flight together.
// out [rows][128]; a row with no partial is all zeros.
__global__ void __launch_bounds__(256) cp_combine_kernel(const float* __restrict__ partials,
                                                         int world, int64_t rows,
                                                         float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= rows) return;
  float M = -INFINITY;
  for (int w0 = 0; w0 < world; w0 += 32) {
    const int w = w0 + lane;
    if (w < world) {
      const float* p = partials + (int64_t(w) * rows + row) * kPartStride;
      if (p[1] > 0.f) M = fmaxf(M, p[0]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float Ls = 0.f;
  if (M != -INFINITY) {
#pragma unroll 4
    for (int w = 0; w < world; ++w) {
      const float* p = partials + (int64_t(w) * rows + row) * kPartStride;
      const float l = p[1];
      const float e = l > 0.f ? exp2f(p[0] - M) : 0.f;
      const float4 a = *reinterpret_cast<const float4*>(p + 4 + 4 * lane);
      Ls = fmaf(l, e, Ls);
      acc.x = fmaf(a.x, e, acc.x);
      acc.y = fmaf(a.y, e, acc.y);
      acc.z = fmaf(a.z, e, acc.z);
      acc.w = fmaf(a.w, e, acc.w);
    }
  }
  const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
  *reinterpret_cast<float4*>(out + row * kD + 4 * lane) =
      make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

cudaError_t launch_cp_combine(const float* partials, int world, int64_t rows, float* out,
                              cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const int64_t blocks = (rows * 32 + 255) / 256;
  cp_combine_kernel<<<unsigned(blocks), 256, 0, stream>>>(partials, world, rows, out);
  return cudaGetLastError();
}

}  // namespace adamas
