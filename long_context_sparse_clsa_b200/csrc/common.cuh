// Device helpers shared by the CLSA kernels (sm_100a).
//
// Everything here is hand-written: inline PTX for cp.async, ldmatrix and the
// bf16 mma, an order-preserving float key for the radix select, the workspace
// error word, and an inter-CTA barrier whose wait is bounded in time.
#pragma once

#include <cstdint>
#include <utility>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/clsa.h"

namespace clsa {

// ---------------------------------------------------------------------------
// workspace header: [0] error code (u32), [8] detail (i64); op regions from 256
// ---------------------------------------------------------------------------
constexpr size_t kWsHeader = 256;
constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bound on every inter-CTA wait: 200 ms of globaltimer.  A correct launch waits
// microseconds; running out records CLSA_ERR_TIMEOUT and the CTA returns.
constexpr unsigned long long kWaitLimitNs = 200ull * 1000ull * 1000ull;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_error(void* ws, uint32_t code, long long detail) {
  uint32_t* w = reinterpret_cast<uint32_t*>(ws);
  if (atomicCAS(w, 0u, code) == 0u) {
    *reinterpret_cast<volatile long long*>(reinterpret_cast<char*>(ws) + 8) = detail;
  }
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Barrier among `nblocks` co-resident CTAs sharing state[0] (arrivals) and
// state[1] (generation).  The arrival count returns to zero each time, so the
// state is reusable by the next launch without clearing.  Returns false (and
// records CLSA_ERR_TIMEOUT with `site`) if the wait ran out; every thread of
// the CTA gets the same answer.
__device__ __forceinline__ bool group_barrier(uint32_t* state, uint32_t nblocks, void* ws, int site) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    if (nblocks > 1) {
      const uint32_t gen = ld_acquire_gpu(state + 1);
      __threadfence();
      const uint32_t arrived = atom_add_acq_rel_gpu(state, 1u);
      if (arrived == nblocks - 1) {
        atomicExch(state, 0u);
        __threadfence();
        st_release_gpu(state + 1, gen + 1u);
      } else {
        const unsigned long long t0 = globaltimer_ns();
        while (ld_acquire_gpu(state + 1) == gen) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            record_error(ws, CLSA_ERR_TIMEOUT, site);
            ok = 0;
            break;
          }
          __nanosleep(32);
        }
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

__device__ __forceinline__ void red_add_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Count-up barrier among `n` co-resident CTAs: `state` counts arrivals (a
// fire-and-forget release add after the CTA's bar.sync, which orders every thread's
// earlier writes before it) and every CTA polls it until it reaches n: one L2 round
// trip after the last arrival.  The word is used once per launch; the caller returns it
// to zero once no CTA polls it any more.  Bounded wait: false (and CLSA_ERR_TIMEOUT
// with `site`) if it runs out.
__device__ __forceinline__ bool count_barrier(uint32_t* state, uint32_t n, void* ws, int site) {
  __shared__ int s_ok2;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    if (n > 1) {
      red_add_release_gpu(state, 1u);
      if (ld_acquire_gpu(state) < n) {
        const unsigned long long t0 = globaltimer_ns();
        while (ld_acquire_gpu(state) < n) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            record_error(ws, CLSA_ERR_TIMEOUT, site);
            ok = 0;
            break;
          }
        }
      }
    }
    s_ok2 = ok;
  }
  __syncthreads();
  return s_ok2 != 0;
}

// ---------------------------------------------------------------------------
// order-preserving key: larger float -> larger unsigned key; -0.0 == +0.0
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------------------
// bf16 / f32 element access
// ---------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

__device__ __forceinline__ void unpack_bf16x2(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xFFFF0000u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// streaming 16-byte load that does not allocate in L1
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// ---------------------------------------------------------------------------
// cp.async / ldmatrix / mma (sm_80+ forms, valid on sm_100a)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte async copy global -> shared; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async_16(void* smem, const void* gmem, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(src_bytes) : "memory");
}
// 4-byte async copy global -> shared (through L1)
__device__ __forceinline__ void cp_async_4(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldmatrix_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                            const void* smem_row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(smem_u32(smem_row)));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                                  const void* smem_row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(smem_u32(smem_row)));
}

// D(16x8 f32) += A(16x16 bf16, row) * B(16x8 bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// mbarrier + 1-D bulk copy (TMA engine, no tensor map, no multicast)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait for phase `parity` of `bar`; false once kWaitLimitNs has passed.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}
// As mbar_wait, but each poll lets the hardware suspend the thread (up to ~4 us) until
// the phase completes, so a waiting warp leaves its scheduler's issue slots to others.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(4000u) : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait_sleep(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait_sleep(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}
// Non-suspending probe of phase `parity` of `bar`.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// Warp-wide bounded wait: lane 0 polls (try_wait, which may suspend it), the others wait
// at the warp barrier, then every lane observes the completed phase itself.  Call with the
// whole warp converged; returns the same value in every lane.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity) {
  uint32_t ok = 1;
  if ((threadIdx.x & 31) == 0 && !mbar_try_wait(bar, parity)) {  // try_wait may suspend: no busy spin
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        ok = 0;
        break;
      }
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) ok = mbar_test_wait(bar, parity) ? 1u : 0u;  // completed: true at once, with ordering
  return __all_sync(0xffffffffu, ok != 0);
}
// As mbar_wait_warp, but lane 0 spins on test_wait (never suspends): for short waits
// (an MMA of a few hundred cycles) where a suspended poller would wake late.
__device__ __forceinline__ bool mbar_spin_warp(uint64_t* bar, uint32_t parity) {
  uint32_t ok = 1;
  if ((threadIdx.x & 31) == 0 && !mbar_test_wait(bar, parity)) {
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_test_wait(bar, parity)) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        ok = 0;
        break;
      }
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) ok = mbar_test_wait(bar, parity) ? 1u : 0u;
  return __all_sync(0xffffffffu, ok != 0);
}
// bulk prefetch of [src, src + bytes) into L2 (src 16-byte aligned, bytes % 16 == 0)
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// global -> shared bulk copy completing on `bar` (dst, src 16-byte aligned, bytes % 16 == 0)
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 2^x by the hardware approximation (ex2.approx.ftz: one special-function op; 2^-inf = 0,
// subnormal results flush to 0)
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// programmatic dependent launch: a kernel launched with launch_pdl may be scheduled while
// the previous kernel on the stream still runs; it must call pdl_enter() before touching
// global memory, which waits for that kernel to complete with its writes visible and then
// lets the next kernel be scheduled in turn.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace clsa
