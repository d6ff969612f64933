// k_gather.cu -- S2, active KV construction (WorldAttention §3.2 "Active KV
// construction"; summary step 4): the selected pool pages are copied, in order,
// into one contiguous K_active / V_active buffer.  A bit-exact, HBM-bound copy:
// 16-byte loads with four in flight per thread, streaming stores, and a grid of a
// few CTAs per SM per (page, K/V) pair.
#include "wa_internal.h"

namespace wa {
namespace {

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
__device__ __forceinline__ void st_stream(uint4* p, const uint4& v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};"
               ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

__global__ void __launch_bounds__(256)
k_gather(const uint4* __restrict__ kp, const uint4* __restrict__ vp, int n_pages, size_t n16,
         const int32_t* __restrict__ sel, uint4* __restrict__ ka, uint4* __restrict__ va,
         uint32_t* err) {
  const int s = blockIdx.y;
  const int page = sel[s];
  if (page < 0 || page >= n_pages) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0) atomicOr(err, WA_DEVERR_PAGE_ID);
    return;
  }
  const uint4* src = (blockIdx.z ? vp : kp) + static_cast<size_t>(page) * n16;
  uint4* dst = (blockIdx.z ? va : ka) + static_cast<size_t>(s) * n16;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    const uint4 a = ld_stream(src + i), b = ld_stream(src + i + stride);
    const uint4 c = ld_stream(src + i + 2 * stride), d = ld_stream(src + i + 3 * stride);
    st_stream(dst + i, a);
    st_stream(dst + i + stride, b);
    st_stream(dst + i + 2 * stride, c);
    st_stream(dst + i + 3 * stride, d);
  }
  for (; i < n16; i += stride) st_stream(dst + i, ld_stream(src + i));
}

__global__ void __launch_bounds__(256)
k_copy16(const uint4* __restrict__ src, uint4* __restrict__ dst, size_t n16) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16; i += stride)
    st_stream(dst + i, ld_stream(src + i));
}

// Row permutation (cube-tile token order, WorldAttention Appendix A.1.3): one warp
// per row, lanes striding over the row's 16-byte vectors with four loads in flight;
// the warps stride over the rows.  inverse == 0 gathers dst[n] = src[perm[n]],
// inverse != 0 scatters dst[perm[n]] = src[n].
__global__ void __launch_bounds__(256)
k_permute_rows(const uint4* __restrict__ src, uint4* __restrict__ dst,
               const int32_t* __restrict__ perm, int n_rows, size_t n16, int inverse,
               uint32_t* err) {
  const int lane = threadIdx.x & 31;
  const int n_warps = static_cast<int>((gridDim.x * blockDim.x) >> 5);
  for (int n = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5); n < n_rows;
       n += n_warps) {
    const int j = perm[n];
    if (j < 0 || j >= n_rows) {
      if (lane == 0) atomicOr(err, WA_DEVERR_ROW_ID);
      continue;
    }
    const uint4* a = src + static_cast<size_t>(inverse ? n : j) * n16;
    uint4* b = dst + static_cast<size_t>(inverse ? j : n) * n16;
    size_t i = lane;
    for (; i + 96 < n16; i += 128) {
      const uint4 x0 = ld_stream(a + i), x1 = ld_stream(a + i + 32);
      const uint4 x2 = ld_stream(a + i + 64), x3 = ld_stream(a + i + 96);
      st_stream(b + i, x0);
      st_stream(b + i + 32, x1);
      st_stream(b + i + 64, x2);
      st_stream(b + i + 96, x3);
    }
    for (; i < n16; i += 32) st_stream(b + i, ld_stream(a + i));
  }
}

}  // namespace

wa_status launch_permute_rows(const void* src, void* dst, const int32_t* perm, int n_rows,
                              size_t row_bytes, int inverse, uint32_t* err, cudaStream_t st) {
  size_t blocks = (static_cast<size_t>(n_rows) + 7) / 8;   // eight warps (rows) per CTA
  if (blocks > 8 * 148) blocks = 8 * 148;
  k_permute_rows<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), perm, n_rows, row_bytes / 16,
      inverse, err);
  return check_launch("permute_rows");
}

wa_status launch_copy16(const void* src, void* dst, size_t n16, cudaStream_t st) {
  size_t blocks = (n16 + 1023) / 1024;
  if (blocks > 8 * 148) blocks = 8 * 148;
  if (blocks < 1) blocks = 1;
  k_copy16<<<static_cast<unsigned>(blocks), 256, 0, st>>>(static_cast<const uint4*>(src),
                                                          static_cast<uint4*>(dst), n16);
  return check_launch("copy16");
}

wa_status launch_gather(const void* k_pool, const void* v_pool, int n_pages, size_t page_bytes,
                        const int32_t* sel, int K_p, void* k_act, void* v_act, uint32_t* err,
                        cudaStream_t st) {
  const size_t n16 = page_bytes / 16;
  int per = (8 * 148) / (2 * K_p);
  if (per < 1) per = 1;
  const size_t need = (n16 + 1023) / 1024;  // at least ~4 vectors per thread
  if (static_cast<size_t>(per) > need) per = static_cast<int>(need < 1 ? 1 : need);
  dim3 grid(per, K_p, 2);
  k_gather<<<grid, 256, 0, st>>>(static_cast<const uint4*>(k_pool),
                                 static_cast<const uint4*>(v_pool), n_pages, n16, sel,
                                 static_cast<uint4*>(k_act), static_cast<uint4*>(v_act), err);
  return check_launch("gather");
}

}  // namespace wa
