// kv_stream.cuh -- the stage decomposition shared by the streaming-ring K/V kernels
// (quantization and calibration statistics of a [B, H, S, D] cache of 16-bit elements).
//
// A stage is 32 KB of the cache: kv_ring_rows(D) = 16384 / D whole rows of one (b, h) block,
// contiguous in memory.  Stages are taken in (tensor, h, b, chunk) order and every CTA of a
// one-wave grid walks a contiguous range of them, so it meets at most a couple of heads (the
// per-channel tables change only with h).  Thread 0 streams the range through a ring of KVR_NS
// shared-memory slots with bulk asynchronous copies (mbarrier completion, never multicast).
// Piece p (16 bytes = 8 channels) of a stage sits at p*16 in its slot; with D/8 a power of two
// dividing the 256 threads, thread t's pieces t + 256k all hold channel group t mod (D/8).
// Measured on [8, 96, 2048, 128] bf16 quantization: 32 KB stages three deep with two CTAs per
// SM stream at 89% of the HBM copy rate, 16 KB stages six deep at 74% (the same bytes in flight,
// twice the per-stage barriers and waits); one CTA per SM with deeper rings ran slower still.
#pragma once

#include "common.cuh"

namespace rptq {

constexpr int KVR_THREADS = 256;
constexpr uint32_t KVR_STAGE = 32768;
constexpr int KVR_PIECES = KVR_STAGE / 16;
constexpr int KVR_PPT = KVR_PIECES / KVR_THREADS;
constexpr int KVR_NS = 3;
__host__ __device__ constexpr int kv_ring_rows(int D) { return (int)(KVR_STAGE / 2) / D; }

// The ring kernels' shape rule: 16-bit elements, D/8 a power of two dividing the 256 threads,
// whole stages per (b, h) block, and stage counts (two tensors) that stay in int.
inline bool kv_ring_shape_ok(int B, int H, int64_t S, int D, int esize)
{
    if (esize != 2 || D < 8 || D % 8 != 0 || D > 2048) return false;
    const int npr = D / 8;
    if ((npr & (npr - 1)) != 0) return false;
    const int64_t sr = kv_ring_rows(D);
    if (S % sr != 0) return false;
    return (int64_t)B * H * (S / sr) * 2 < 0x7fffffffLL;
}

// A stage's place in (tensor, h, b, chunk) order, advanced without divisions.
struct KvStagePos {
    int ti, h, b, chunk;
    __device__ __forceinline__ void set(int64_t j, int64_t per_t, int B, int SPB)
    {
        ti = (int)(j / per_t);
        int64_t r = j - ti * per_t;
        const int64_t per_h = (int64_t)B * SPB;
        h = (int)(r / per_h);
        r -= h * per_h;
        b = (int)(r / SPB);
        chunk = (int)(r - (int64_t)b * SPB);
    }
    __device__ __forceinline__ void advance(int B, int H, int SPB)
    {
        if (++chunk == SPB) {
            chunk = 0;
            if (++b == B) {
                b = 0;
                if (++h == H) {
                    h = 0;
                    ++ti;
                }
            }
        }
    }
    // stage number within its tensor in memory order (b, h, chunk)
    __device__ __forceinline__ int64_t mem_index(int H, int SPB) const { return ((int64_t)b * H + h) * SPB + chunk; }
};

}  // namespace rptq
