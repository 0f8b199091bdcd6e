// Selector: gather the selected K/V rows once into a compact buffer
// (zhichai.net "CLSA Explained", CLSA: Sharing the Index Across Layers: later
// layers gather KV by the shared index; here the gather happens once for all).
//
// One warp per selected token copies its K and V rows (Hkv * d * elem bytes,
// contiguous in the [n][Hkv][d] cache) with 16-byte loads and stores, up to 4 K and 4 V
// loads per lane in flight before the stores (a 4 KiB bf16 row pair per warp at once).  An index
// outside [0, n_max) is never dereferenced: the row is zero-filled and
// CLSA_ERR_BAD_INDEX (detail = b * 2^32 + i) is recorded.
#include "common.cuh"
#include "kernels.h"

namespace clsa {

namespace {

__global__ void __launch_bounds__(256) gather_kv_kernel(const uint4* __restrict__ K, const uint4* __restrict__ V,
                                                        const int32_t* __restrict__ idx,
                                                        const int32_t* __restrict__ count, int n_max, int k,
                                                        int row_vec, uint4* __restrict__ KS,
                                                        uint4* __restrict__ VS, void* ws_header) {
  const int b = blockIdx.y;
  const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= k || i >= count[b]) return;  // count is clamped to k by this test
  const int t = idx[(size_t)b * k + i];
  uint4* dk = KS + ((size_t)b * k + i) * row_vec;
  uint4* dv = VS + ((size_t)b * k + i) * row_vec;
  if (t < 0 || t >= n_max) {
    if (lane == 0) record_error(ws_header, CLSA_ERR_BAD_INDEX, ((long long)b << 32) | (unsigned)i);
    for (int c = lane; c < row_vec; c += 32) {
      dk[c] = make_uint4(0, 0, 0, 0);
      dv[c] = make_uint4(0, 0, 0, 0);
    }
    return;
  }
  const uint4* sk = K + ((size_t)b * n_max + t) * row_vec;
  const uint4* sv = V + ((size_t)b * n_max + t) * row_vec;
  // every load of a batch is issued before its stores: 2 kU 16-byte loads in flight per lane
  constexpr int kU = 4;
  for (int c0 = lane; c0 < row_vec; c0 += 32 * kU) {
    uint4 a[kU], v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int c = c0 + 32 * u;
      if (c < row_vec) {
        a[u] = ld_stream_v4(sk + c);
        v[u] = ld_stream_v4(sv + c);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int c = c0 + 32 * u;
      if (c < row_vec) {
        dk[c] = a[u];
        dv[c] = v[u];
      }
    }
  }
}

}  // namespace

cudaError_t launch_gather_kv(const void* K, const void* V, const int32_t* idx, const int32_t* count, int B,
                             int n_max, int k, int Hkv, int d, clsa_dtype dt, void* K_S, void* V_S,
                             void* ws_header, cudaStream_t s) {
  const int esz = dt == CLSA_BF16 ? 2 : 4;
  const int row_vec = Hkv * d * esz / 16;
  dim3 grid((k + 7) / 8, B);
  gather_kv_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(K), static_cast<const uint4*>(V), idx, count,
                                        n_max, k, row_vec, static_cast<uint4*>(K_S), static_cast<uint4*>(V_S),
                                        ws_header);
  launches_add(1, s);
  return cudaGetLastError();
}

}  // namespace clsa
