// stage.cu -- one launch that copies up to kMaxRanges byte ranges, with the
// loads and stores issued by the SMs.
//
// A decode step's inputs are a handful of small tensors (the 2.9B shape:
// 256 KiB of absorbed queries, 32 KiB of RoPE queries, 8 KiB of block table,
// 64 bytes of lengths).  Copied from pinned host memory by the DMA engine,
// each tensor pays the copy engine's setup latency; read by the SMs straight
// from the mapped pinned pages, all of them cross PCIe in one launch with
// thousands of 16-byte reads in flight.  Nothing here is specific to the
// method: it is the host-to-device leg of a serving step.
#include "common.cuh"
#include "kernels.h"

namespace mlra {
namespace {

constexpr int kStageThreads = 256;
constexpr int kUnroll = 4;  // 16-byte units in flight per thread

__global__ void __launch_bounds__(kStageThreads)
copy_ranges_kernel(const CopyRanges r) {
    // 16-byte units of every range whose ends are 16-byte aligned; the
    // ranges' byte tails (size % 16) are copied by the last CTA
    const size_t stride = (size_t)gridDim.x * kStageThreads;
    const size_t tid = (size_t)blockIdx.x * kStageThreads + threadIdx.x;
    for (int k = 0; k < r.count; ++k) {
        const uint4* src = static_cast<const uint4*>(r.src[k]);
        uint4* dst = static_cast<uint4*>(r.dst[k]);
        const size_t units = r.bytes[k] / 16;
        size_t u = tid;
        for (; u + (kUnroll - 1) * stride < units; u += kUnroll * stride) {
            uint4 v[kUnroll];
#pragma unroll
            for (int i = 0; i < kUnroll; ++i) v[i] = __ldcv(src + u + i * stride);
#pragma unroll
            for (int i = 0; i < kUnroll; ++i) dst[u + i * stride] = v[i];
        }
        for (; u < units; u += stride) dst[u] = __ldcv(src + u);
        if (blockIdx.x == gridDim.x - 1) {
            const size_t tail = r.bytes[k] % 16;
            if (threadIdx.x < tail)
                static_cast<uint8_t*>(r.dst[k])[units * 16 + threadIdx.x] =
                    static_cast<const uint8_t*>(r.src[k])[units * 16 + threadIdx.x];
        }
    }
}

}  // namespace

cudaError_t launch_copy_ranges(const CopyRanges& r, int sms, cudaStream_t stream) {
    size_t units = 0;
    for (int k = 0; k < r.count; ++k) units += r.bytes[k] / 16;
    // enough threads that every unit of the largest batch of reads is in
    // flight at once, at most two CTAs per SM
    const size_t want = (units + (size_t)kStageThreads * kUnroll - 1) / ((size_t)kStageThreads * kUnroll);
    const int grid = (int)(want < 1 ? 1 : (want > (size_t)2 * sms ? (size_t)2 * sms : want));
    copy_ranges_kernel<<<grid, kStageThreads, 0, stream>>>(r);
    return cudaGetLastError();
}

}  // namespace mlra
