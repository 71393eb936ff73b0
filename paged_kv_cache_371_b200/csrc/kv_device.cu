// Device-side helpers of the paged KV library: the per-device error word, the
// cache-append scatter and the copy-on-write block copy.
//
// Cache append: each decode step writes the new token's K and V into the slot
// the host reserved for it ("LLM 推理优化：KV Cache、PagedAttention 与量化"
// §2.3 (1): blocks are filled on write).  Block copy: the copy-on-write step of
// §2.3 (2) of the same page (the block a beam writes into is copied first).
// Both are plain byte moves: 16-byte vector loads/stores, fully coalesced
// within each (token, head) row and each block.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/paged_kv.h"
#include "kv_device.h"
#include "kv_ptx.cuh"
#include "kv_status.h"

namespace {

__device__ int g_kv_error_word;

constexpr int kMaxDevices = 64;
int* g_word_ptr[kMaxDevices];
std::mutex g_word_mu;

__global__ void append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                              const int64_t* __restrict__ slot_mapping, uint4* __restrict__ k_pool,
                              uint4* __restrict__ v_pool, int32_t T, int32_t Hkv,
                              int32_t chunks_per_row, int32_t bs, int64_t num_slots, int* err)
{
    // a decode-attention launch that follows may start its set-up (it waits
    // for this grid before it reads the pools)
    pkv::pdl_launch_dependents();
    // one thread per 16-byte chunk of one (token, head) row, K and V together
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t per_tok = (int64_t)Hkv * chunks_per_row;
    if (i >= (int64_t)T * per_tok) return;
    const int32_t t = (int32_t)(i / per_tok);
    const int32_t rem = (int32_t)(i % per_tok);
    const int32_t h = rem / chunks_per_row;
    const int32_t c = rem % chunks_per_row;
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (rem == 0) atomicOr(err, KV_DEV_BAD_SLOT);
        return;
    }
    const int64_t blk = slot / bs;
    const int32_t off = (int32_t)(slot % bs);
    const int64_t dst = ((blk * Hkv + h) * bs + off) * chunks_per_row + c;
    k_pool[dst] = __ldg(k_new + i);
    v_pool[dst] = __ldg(v_new + i);
}

__global__ void copy_blocks_kernel(uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                   const int32_t* __restrict__ pairs, int32_t n,
                                   int64_t chunks_per_block, int32_t num_blocks, int* err,
                                   int64_t k_chunks_per_block)
{
    const int32_t pair = blockIdx.y;
    const int32_t src = __ldg(pairs + 2 * pair);
    const int32_t dst = __ldg(pairs + 2 * pair + 1);
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(err, KV_DEV_BAD_BLOCK);
        return;
    }
    // K blocks may be smaller than V blocks (int8 codes): k_chunks_per_block
    const uint4* ks = k_pool + (int64_t)src * k_chunks_per_block;
    const uint4* vs = v_pool + (int64_t)src * chunks_per_block;
    uint4* kd = k_pool + (int64_t)dst * k_chunks_per_block;
    uint4* vd = v_pool + (int64_t)dst * chunks_per_block;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < chunks_per_block;
         c += (int64_t)gridDim.x * blockDim.x) {
        if (c < k_chunks_per_block) kd[c] = ks[c];
        vd[c] = vs[c];
    }
}

// Quantised K ("大模型推理加速：从 KV Cache 到投机采样的工程实践" §"KV Cache量化":
// keys per channel; "LLM 推理优化：KV Cache、PagedAttention 与量化" §4.2: keys
// at low bit width per channel, values FP16): code = clamp(rint(k / s), -128,
// 127) with one fp32 scale s per (KV head, channel); correctly rounded fp32
// division, round half to even.  One thread per 8 channels of one (token,
// head) row: 8 codes (8 bytes) of K, 16 bytes of V.
__global__ void append_q8k_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                  const int64_t* __restrict__ slot_mapping,
                                  const float* __restrict__ k_scales, uint2* __restrict__ kq_pool,
                                  uint4* __restrict__ v_pool, int32_t T, int32_t Hkv,
                                  int32_t chunks_per_row, int32_t bs, int64_t num_slots, int* err)
{
    pkv::pdl_launch_dependents();  // as in append_kernel
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t per_tok = (int64_t)Hkv * chunks_per_row;
    if (i >= (int64_t)T * per_tok) return;
    const int32_t t = (int32_t)(i / per_tok);
    const int32_t rem = (int32_t)(i % per_tok);
    const int32_t h = rem / chunks_per_row;
    const int32_t c = rem % chunks_per_row;
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (rem == 0) atomicOr(err, KV_DEV_BAD_SLOT);
        return;
    }
    const int64_t blk = slot / bs;
    const int32_t off = (int32_t)(slot % bs);
    const int64_t dst = ((blk * Hkv + h) * bs + off) * chunks_per_row + c;
    const uint4 kv = __ldg(k_new + i);
    const float* sc = k_scales + ((int64_t)h * chunks_per_row + c) * 8;
    const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
    uint32_t packed[2] = {0u, 0u};
    bool bad = false;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const uint32_t w = kw[e >> 1];
        const float k = __half2float(__ushort_as_half((unsigned short)(e & 1 ? w >> 16 : w & 0xffff)));
        const float s = __ldg(sc + e);
        int code = 0;
        if (s > 0.f && s <= 3.402823466e38f) {
            const float r = rintf(__fdiv_rn(k, s));
            code = r != r ? 0 : (int)fminf(fmaxf(r, -128.f), 127.f);  // NaN key: code 0
        } else {
            bad = true;
        }
        packed[e >> 2] |= (uint32_t)(code & 0xff) << (8 * (e & 3));
    }
    if (bad) atomicOr(err, KV_DEV_BAD_SCALE);
    kq_pool[dst] = make_uint2(packed[0], packed[1]);
    v_pool[dst] = __ldg(v_new + i);
}

// Calibration scales: s[h][d] = max_t |k[t][h][d]| / 127 (1 for an all-zero
// channel); one thread per (head, channel), over all T tokens.
__global__ void k_scales_kernel(const __half* __restrict__ k, int64_t T, int32_t Hkv, int32_t D,
                                float* __restrict__ scales)
{
    const int32_t i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= Hkv * D) return;
    float amax = 0.f;
    for (int64_t t = 0; t < T; ++t) amax = fmaxf(amax, fabsf(__half2float(k[t * Hkv * D + i])));
    scales[i] = amax > 0.f ? __fdiv_rn(amax, 127.f) : 1.f;
}

// Swap staging: [2 (K, V)][n][block chunks].  to_pool = 0: pool blocks ids[i]
// -> staging row i; 1: the reverse.  Out-of-range ids are skipped and flagged.
__global__ void swap_blocks_kernel(uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                   const int32_t* __restrict__ ids, int32_t n,
                                   uint4* __restrict__ staging, int64_t chunks_per_block,
                                   int32_t num_blocks, int to_pool, int* err)
{
    const int32_t i = blockIdx.y;
    const int32_t b = __ldg(ids + i);
    if (b < 0 || b >= num_blocks) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(err, KV_DEV_BAD_BLOCK);
        return;
    }
    uint4* kp = k_pool + (int64_t)b * chunks_per_block;
    uint4* vp = v_pool + (int64_t)b * chunks_per_block;
    uint4* ks = staging + (int64_t)i * chunks_per_block;
    uint4* vs = staging + ((int64_t)n + i) * chunks_per_block;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < chunks_per_block;
         c += (int64_t)gridDim.x * blockDim.x) {
        if (to_pool) {
            kp[c] = ks[c];
            vp[c] = vs[c];
        } else {
            ks[c] = kp[c];
            vs[c] = vp[c];
        }
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int swap_impl(void* k_pool, void* v_pool, const int32_t* ids, int32_t n, void* staging, void* host,
              int32_t Hkv, int32_t head_dim, int32_t block_size, int32_t num_blocks, int to_pool,
              void* stream, const char* name)
{
    if (n < 0 || n > 65535 || Hkv <= 0 || head_dim <= 0 || head_dim % 8 != 0 || block_size <= 0 ||
        num_blocks <= 0)
        return kv_fail(KV_ERR_INVALID, name);
    if (n == 0) return KV_OK;
    if (!k_pool || !v_pool || !ids || !staging) return kv_fail(KV_ERR_INVALID, name);
    if (!aligned16(k_pool) || !aligned16(v_pool) || !aligned16(staging))
        return kv_fail(KV_ERR_INVALID, name);
    int* err = kv_error_word_ptr();
    if (!err) return kv_fail(KV_ERR_CUDA, name);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t cpb = (int64_t)Hkv * block_size * head_dim / 8;
    const size_t bytes = (size_t)2 * n * cpb * 16;
    int rc;
    if (to_pool && host &&
        (rc = kv_cuda_check(cudaMemcpyAsync(staging, host, bytes, cudaMemcpyHostToDevice, st), name)) != KV_OK)
        return rc;
    const int threads = 256;
    int64_t bx = (cpb + threads - 1) / threads;
    if (bx > 64) bx = 64;
    swap_blocks_kernel<<<dim3((unsigned)bx, (unsigned)n), threads, 0, st>>>(
        static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), ids, n, static_cast<uint4*>(staging),
        cpb, num_blocks, to_pool, err);
    if ((rc = kv_cuda_check(cudaGetLastError(), name)) != KV_OK) return rc;
    if (!to_pool && host)
        return kv_cuda_check(cudaMemcpyAsync(host, staging, bytes, cudaMemcpyDeviceToHost, st), name);
    return KV_OK;
}

}  // namespace

int* kv_error_word_ptr()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_word_mu);
    if (!g_word_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kv_error_word) != cudaSuccess) return nullptr;
        g_word_ptr[dev] = static_cast<int*>(p);
    }
    return g_word_ptr[dev];
}

int kv_cuda_check(cudaError_t e, const char* where)
{
    if (e == cudaSuccess) return KV_OK;
    static thread_local char buf[256];
    snprintf(buf, sizeof(buf), "%s: %s", where, cudaGetErrorString(e));
    return kv_fail(KV_ERR_CUDA, buf);
}

extern "C" {

int paged_kv_append(const void* k_new, const void* v_new, const int64_t* slot_mapping,
                    void* k_pool, void* v_pool, int32_t T, int32_t Hkv, int32_t head_dim,
                    int32_t block_size, int32_t num_blocks, void* stream)
{
    if (T < 0 || Hkv <= 0 || head_dim <= 0 || head_dim % 8 != 0 || block_size <= 0 ||
        num_blocks <= 0)
        return kv_fail(KV_ERR_INVALID, "paged_kv_append: bad sizes");
    if (T == 0) return KV_OK;
    if (!k_new || !v_new || !slot_mapping || !k_pool || !v_pool)
        return kv_fail(KV_ERR_INVALID, "paged_kv_append: null pointer");
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) || !aligned16(v_pool))
        return kv_fail(KV_ERR_INVALID, "paged_kv_append: buffers must be 16-byte aligned");
    int* err = kv_error_word_ptr();
    if (!err) return kv_fail(KV_ERR_CUDA, "paged_kv_append: no device error word");
    const int32_t cpr = head_dim / 8;
    const int64_t total = (int64_t)T * Hkv * cpr;
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    append_kernel<<<(unsigned)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), slot_mapping,
        static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), T, Hkv, cpr, block_size,
        (int64_t)num_blocks * block_size, err);
    return kv_cuda_check(cudaGetLastError(), "paged_kv_append");
}


static int copy_blocks_impl(void* k_pool, void* v_pool, const int32_t* pairs, int32_t n,
                            int32_t Hkv, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                            void* stream, bool k_int8)
{
    if (n < 0 || Hkv <= 0 || head_dim <= 0 || head_dim % 8 != 0 || block_size <= 0 ||
        num_blocks <= 0 || n > 65535)
        return kv_fail(KV_ERR_INVALID, "paged_kv_copy_blocks: bad sizes");
    if (n == 0) return KV_OK;
    if (!k_pool || !v_pool || !pairs)
        return kv_fail(KV_ERR_INVALID, "paged_kv_copy_blocks: null pointer");
    if (!aligned16(k_pool) || !aligned16(v_pool))
        return kv_fail(KV_ERR_INVALID, "paged_kv_copy_blocks: pools must be 16-byte aligned");
    int* err = kv_error_word_ptr();
    if (!err) return kv_fail(KV_ERR_CUDA, "paged_kv_copy_blocks: no device error word");
    const int64_t cpb = (int64_t)Hkv * block_size * head_dim / 8;
    const int threads = 256;
    int64_t bx = (cpb + threads - 1) / threads;
    if (bx > 64) bx = 64;
    dim3 grid((unsigned)bx, (unsigned)n);
    copy_blocks_kernel<<<grid, threads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), pairs, n, cpb, num_blocks, err,
        k_int8 ? cpb / 2 : cpb);
    return kv_cuda_check(cudaGetLastError(), "paged_kv_copy_blocks");
}

int paged_kv_copy_blocks(void* k_pool, void* v_pool, const int32_t* pairs, int32_t n, int32_t Hkv,
                         int32_t head_dim, int32_t block_size, int32_t num_blocks, void* stream)
{
    return copy_blocks_impl(k_pool, v_pool, pairs, n, Hkv, head_dim, block_size, num_blocks, stream,
                            false);
}

int paged_kv_copy_blocks_q8k(void* kq_pool, void* v_pool, const int32_t* pairs, int32_t n,
                             int32_t Hkv, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                             void* stream)
{
    if (head_dim % 16 != 0) return kv_fail(KV_ERR_INVALID, "paged_kv_copy_blocks_q8k: bad head_dim");
    return copy_blocks_impl(kq_pool, v_pool, pairs, n, Hkv, head_dim, block_size, num_blocks, stream,
                            true);
}

int paged_kv_append_q8k(const void* k_new, const void* v_new, const int64_t* slot_mapping,
                        const float* k_scales, void* kq_pool, void* v_pool, int32_t T, int32_t Hkv,
                        int32_t head_dim, int32_t block_size, int32_t num_blocks, void* stream)
{
    if (T < 0 || Hkv <= 0 || head_dim <= 0 || head_dim % 8 != 0 || block_size <= 0 ||
        num_blocks <= 0)
        return kv_fail(KV_ERR_INVALID, "paged_kv_append_q8k: bad sizes");
    if (T == 0) return KV_OK;
    if (!k_new || !v_new || !slot_mapping || !k_scales || !kq_pool || !v_pool)
        return kv_fail(KV_ERR_INVALID, "paged_kv_append_q8k: null pointer");
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(kq_pool) || !aligned16(v_pool) ||
        (reinterpret_cast<uintptr_t>(k_scales) & 3u))
        return kv_fail(KV_ERR_INVALID, "paged_kv_append_q8k: misaligned buffer");
    int* err = kv_error_word_ptr();
    if (!err) return kv_fail(KV_ERR_CUDA, "paged_kv_append_q8k: no device error word");
    const int32_t cpr = head_dim / 8;
    const int64_t total = (int64_t)T * Hkv * cpr;
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    append_q8k_kernel<<<(unsigned)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), slot_mapping, k_scales,
        static_cast<uint2*>(kq_pool), static_cast<uint4*>(v_pool), T, Hkv, cpr, block_size,
        (int64_t)num_blocks * block_size, err);
    return kv_cuda_check(cudaGetLastError(), "paged_kv_append_q8k");
}

int paged_kv_k_scales(const void* k, int64_t T, int32_t Hkv, int32_t head_dim, float* scales,
                      void* stream)
{
    if (T < 0 || Hkv <= 0 || head_dim <= 0 || !scales || (T > 0 && !k))
        return kv_fail(KV_ERR_INVALID, "paged_kv_k_scales: bad argument");
    const int n = Hkv * head_dim;
    k_scales_kernel<<<(n + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __half*>(k), T, Hkv, head_dim, scales);
    return kv_cuda_check(cudaGetLastError(), "paged_kv_k_scales");
}

int paged_kv_swap_out(const void* k_pool, const void* v_pool, const int32_t* block_ids, int32_t n,
                      void* staging, void* host, int32_t Hkv, int32_t head_dim, int32_t block_size,
                      int32_t num_blocks, void* stream)
{
    return swap_impl(const_cast<void*>(k_pool), const_cast<void*>(v_pool), block_ids, n, staging, host,
                     Hkv, head_dim, block_size, num_blocks, 0, stream, "paged_kv_swap_out: bad argument");
}

int paged_kv_swap_in(void* k_pool, void* v_pool, const int32_t* block_ids, int32_t n, void* staging,
                     const void* host, int32_t Hkv, int32_t head_dim, int32_t block_size,
                     int32_t num_blocks, void* stream)
{
    return swap_impl(k_pool, v_pool, block_ids, n, staging, const_cast<void*>(host), Hkv, head_dim,
                     block_size, num_blocks, 1, stream, "paged_kv_swap_in: bad argument");
}

int kv_device_error(int32_t* word_out, int32_t reset, void* stream)
{
    if (!word_out) return kv_fail(KV_ERR_INVALID, "kv_device_error: null output");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int rc = kv_cuda_check(cudaMemcpyFromSymbolAsync(word_out, g_kv_error_word, sizeof(int32_t), 0,
                                                     cudaMemcpyDeviceToHost, st),
                           "kv_device_error");
    if (rc != KV_OK) return rc;
    if (reset) {
        const int32_t zero = 0;
        rc = kv_cuda_check(cudaMemcpyToSymbolAsync(g_kv_error_word, &zero, sizeof(int32_t), 0,
                                                   cudaMemcpyHostToDevice, st),
                           "kv_device_error");
        if (rc != KV_OK) return rc;
    }
    return kv_cuda_check(cudaStreamSynchronize(st), "kv_device_error");
}

}  // extern "C"
