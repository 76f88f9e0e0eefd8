// Building blocks shared by the tensor-core kernels (sm_100a): shared-memory
// matrix descriptors of tcgen05.mma operands, bounded mbarrier waits, TMA
// loads, tcgen05.commit, and the host-side tensor-map encoder.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cuda_runtime.h>

namespace mxfp4 {
namespace {

// Upper bound on the polls of one mbarrier wait (each poll may suspend the
// thread for a while): a wait that runs out reports failure instead of
// spinning forever.
constexpr long long kWaitLimit = 1ll << 22;
// The waits of the threads that read the accumulator out of tensor memory
// for its completion. A test build defines MXFP4_ACC_WAIT_POLLS to 0, so
// that on a normal input those waits give up at once and the timeout path
// (NaN or zero-scale tiles, the caller's status word, the drains) runs;
// every other wait keeps kWaitLimit.
#ifndef MXFP4_ACC_WAIT_POLLS
#define MXFP4_ACC_WAIT_POLLS (1ll << 22)
#endif
constexpr long long kAccWaitLimit = MXFP4_ACC_WAIT_POLLS;
// Bit the tensor-core kernels OR into the caller's status word when a wait
// ran out (MXFP4_STATUS_WAIT_TIMEOUT of the public header).
constexpr int kStatusWaitTimeout = 1;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Matrix descriptor of a K-major operand in shared memory without swizzle:
// start address, leading byte offset (between 16-byte K columns), stride
// byte offset (between 8-row groups), all in 16-byte units; version 1.
__device__ __forceinline__ uint64_t smem_desc(const void* p, uint32_t lbo,
                                              uint32_t sbo) {
  uint64_t d = (smem_u32(p) >> 4) & 0x3FFFu;
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;
  return d;
}

// Descriptor of a 128-byte-swizzled K-major operand: 8-row groups 1024
// bytes apart; a K step inside the 128-byte swizzle row moves the start
// address by its byte offset (32 bytes = 64 fp4 or 16 bf16 elements).
__device__ __forceinline__ uint64_t smem_desc_sw128(const void* p) {
  uint64_t d = (smem_u32(p) >> 4) & 0x3FFFu;
  d |= uint64_t(1) << 16;                  // leading byte offset (unused)
  d |= uint64_t(1024 >> 4) << 32;          // stride byte offset
  d |= uint64_t(1) << 46;                  // version
  d |= uint64_t(2) << 61;                  // 128-byte swizzle
  return d;
}

__device__ __forceinline__ bool wait_parity(unsigned long long* bar,
                                            uint32_t parity,
                                            long long limit = kWaitLimit) {
  const uint32_t a = smem_u32(bar);
  for (long long i = 0; i < limit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

// wait_parity for threads off the critical path (a producer that runs
// ahead of a slower consumer): between failed polls the thread sleeps, so
// its polls do not take issue slots from the warps doing the work.
constexpr unsigned kPollSleepNs = 128;
__device__ __forceinline__ bool wait_parity_sleep(unsigned long long* bar,
                                                  uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  for (long long i = 0; i < kWaitLimit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
    __nanosleep(kPollSleepNs);
  }
  return false;
}

// wait_parity for a barrier that another role of the CTA feeds: gives up
// as soon as *failed is set (that role timed out and stopped), checking the
// flag every 64 polls; with SLEEP the thread naps between polls as in
// wait_parity_sleep.
template <bool SLEEP>
__device__ __forceinline__ bool wait_parity_or_failed(unsigned long long* bar,
                                                      uint32_t parity, const int* failed) {
  const uint32_t a = smem_u32(bar);
  for (long long i = 0; i < kWaitLimit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
    if ((i & 63) == 63 && *static_cast<const volatile int*>(failed) != 0) return false;
    if (SLEEP) __nanosleep(kPollSleepNs);
  }
  return false;
}

__device__ __forceinline__ void expect_tx(unsigned long long* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x,
                                            int y, unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool failed_flag(const int* f) {
  return *static_cast<const volatile int*>(f) != 0;
}

// Arrive on bar once every tensor-core operation this thread issued so far
// has completed.
__device__ __forceinline__ void commit_to(unsigned long long* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar)));
}

// Thread 0, after the kernel's last __syncthreads: OR the timeout bit into
// the caller's status word if any wait of this CTA ran out.
__device__ __forceinline__ void report_failure(int* status, const int* failed) {
  if (threadIdx.x == 0 && status != nullptr && *static_cast<const volatile int*>(failed) != 0)
    atomicOr(status, kStatusWaitTimeout);
}

// cuTensorMapEncodeTiled through the entry point the runtime hands out (no
// driver library is linked).
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D map over a row-major byte array [rows][row_bytes]: boxes of 128 bytes
// x box_rows, 128-byte swizzle, zero fill outside the array.
inline bool encode_rows_sw128(CUtensorMap* map, const void* base, int64_t rows,
                              int64_t row_bytes, uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cuuint64_t(row_bytes), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(row_bytes)};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace
}  // namespace mxfp4
