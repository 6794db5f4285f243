// K4 (CUDA-core form): indexer token scores for any head subset.
//
//   dense (Eq. 1 of the MISA paper summary, Introduction):
//       I[t,s]    = sum_{j < H}       w[t,j] * ReLU(q[t,j] . k[s])
//   routed (Eq. 9, Methodology section 1):
//       Ihat[t,s] = sum_{j in heads_t} w[t,j] * ReLU(q[t,j] . k[s])
//
// One CTA of 128 threads handles one query row and walks key tiles of 128 tokens,
// one token per thread.  The row's selected query vectors (fp32) and weights sit in
// shared memory and are read as broadcasts; each thread streams its key row in
// 16-byte slices and keeps one fp32 dot-product accumulator per head in registers.
// This is the general form (any head count up to 128, gathered token lists for the
// MISA-dagger fine stage); the tensor-core kernels take over the large shapes.
#include "common.cuh"
#include "internal.h"

namespace misa {
namespace {

constexpr int kTile = 128;

template <int NH>
__global__ void __launch_bounds__(kTile) score_simt_kernel(
    const uint16_t* __restrict__ q, const float* __restrict__ w, const uint4* __restrict__ k,
    const int32_t* __restrict__ heads, int hsel, const int32_t* __restrict__ pos,
    const int32_t* __restrict__ gather_ids, const int32_t* __restrict__ gather_len, int T,
    int H, int64_t L, float* __restrict__ out, int64_t out_stride, int* status, int64_t row0) {
  extern __shared__ __align__(16) float smem[];
  float4* qs = reinterpret_cast<float4*>(smem);           // [NH][32] float4
  float* wsel = smem + NH * kHeadDim;                      // [NH]
  const int64_t row = row0 + blockIdx.y;
  const int64_t n = row / T;
  const int tid = threadIdx.x;
  const bool gather = gather_ids != nullptr;
  int len;
  if (gather) {
    len = (int)min((int64_t)max(gather_len[row], 0), out_stride);
  } else {
    len = prefix_len(pos, row, L, (blockIdx.x == 0 && tid == 0) ? status : nullptr);
  }
  if ((int64_t)blockIdx.x * kTile >= len) return;

  const int nh = heads ? hsel : H;
  for (int r = tid; r < NH; r += kTile) {
    int j = -1;
    if (r < nh) {
      j = heads ? heads[row * hsel + r] : r;
      if (j < 0 || j >= H) {
        if (blockIdx.x == 0) set_status(status, MISA_ERR_BAD_DEVICE_INPUT);
        j = -1;
      }
    }
    wsel[r] = j >= 0 ? w[row * H + j] : 0.f;
  }
  for (int e = tid; e < NH * (kHeadDim / 8); e += kTile) {
    const int r = e / (kHeadDim / 8), c = e % (kHeadDim / 8);
    int j = -1;
    if (r < nh) {
      j = heads ? heads[row * hsel + r] : r;
      if (j < 0 || j >= H) j = -1;
    }
    float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;
    if (j >= 0) {
      const uint4 v = reinterpret_cast<const uint4*>(q + (row * H + j) * kHeadDim)[c];
      lo = make_float4(bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y));
      hi = make_float4(bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w));
    }
    qs[r * 32 + 2 * c] = lo;
    qs[r * 32 + 2 * c + 1] = hi;
  }
  __syncthreads();

  for (int64_t tile = blockIdx.x; tile * kTile < len; tile += gridDim.x) {
    const int i = (int)(tile * kTile) + tid;
    if (i >= len) continue;
    int64_t s = gather ? (int64_t)gather_ids[row * out_stride + i] : (int64_t)i;
    if (s < 0 || s >= L) {   // a gathered id outside the sequence: reported, scored as key 0
      set_status(status, MISA_ERR_BAD_DEVICE_INPUT);
      s = 0;
    }
    const uint4* kr = k + (n * L + s) * 16;
    float acc[NH];
#pragma unroll
    for (int r = 0; r < NH; ++r) acc[r] = 0.f;
#pragma unroll 2
    for (int c = 0; c < kHeadDim / 8; ++c) {
      const uint4 v = kr[c];
      const float f0 = bf16lo(v.x), f1 = bf16hi(v.x), f2 = bf16lo(v.y), f3 = bf16hi(v.y);
      const float f4 = bf16lo(v.z), f5 = bf16hi(v.z), f6 = bf16lo(v.w), f7 = bf16hi(v.w);
#pragma unroll
      for (int r = 0; r < NH; ++r) {
        const float4 a = qs[r * 32 + 2 * c], b = qs[r * 32 + 2 * c + 1];
        float x = acc[r];
        x = fmaf(a.x, f0, x); x = fmaf(a.y, f1, x); x = fmaf(a.z, f2, x); x = fmaf(a.w, f3, x);
        x = fmaf(b.x, f4, x); x = fmaf(b.y, f5, x); x = fmaf(b.z, f6, x); x = fmaf(b.w, f7, x);
        acc[r] = x;
      }
    }
    float sc = 0.f;
#pragma unroll
    for (int r = 0; r < NH; ++r) sc = fmaf(wsel[r], fmaxf(acc[r], 0.f), sc);
    out[row * out_stride + i] = sc;
  }
}

template <int NH>
cudaError_t launch_nh(const uint16_t* q, const float* w, const uint16_t* k, const int32_t* heads,
                      int hsel, const int32_t* pos, const int32_t* gather_ids,
                      const int32_t* gather_len, int rows, int T, int H, int64_t L, float* out,
                      int64_t out_stride, int* status, cudaStream_t st) {
  const size_t smem = (size_t)NH * kHeadDim * sizeof(float) + NH * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(score_simt_kernel<NH>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t span = gather_ids ? out_stride : L;
  int64_t tiles = (span + kTile - 1) / kTile;
  if (tiles > 65535) tiles = 65535;
  for (int64_t row0 = 0; row0 < rows; row0 += 65535) {
    const int64_t nr = rows - row0 < 65535 ? rows - row0 : 65535;
    dim3 grid((unsigned)tiles, (unsigned)nr);
    score_simt_kernel<NH><<<grid, kTile, smem, st>>>(q, w, reinterpret_cast<const uint4*>(k),
                                                    heads, hsel, pos, gather_ids, gather_len, T,
                                                    H, L, out, out_stride, status, row0);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_score_simt(const uint16_t* q, const float* w, const uint16_t* k,
                              const int32_t* heads, int hsel, const int32_t* pos,
                              const int32_t* gather_ids, const int32_t* gather_len,
                              int nseq, int T, int H, int64_t L, float* out,
                              int64_t out_stride, int* status, cudaStream_t st) {
  const int rows = nseq * T;
  const int nh = heads ? hsel : H;
  if (nh <= 8)
    return launch_nh<8>(q, w, k, heads, hsel, pos, gather_ids, gather_len, rows, T, H, L, out,
                        out_stride, status, st);
  if (nh <= 16)
    return launch_nh<16>(q, w, k, heads, hsel, pos, gather_ids, gather_len, rows, T, H, L, out,
                         out_stride, status, st);
  if (nh <= 32)
    return launch_nh<32>(q, w, k, heads, hsel, pos, gather_ids, gather_len, rows, T, H, L, out,
                         out_stride, status, st);
  if (nh <= 64)
    return launch_nh<64>(q, w, k, heads, hsel, pos, gather_ids, gather_len, rows, T, H, L, out,
                         out_stride, status, st);
  return launch_nh<128>(q, w, k, heads, hsel, pos, gather_ids, gather_len, rows, T, H, L, out,
                        out_stride, status, st);
}

}  // namespace misa
