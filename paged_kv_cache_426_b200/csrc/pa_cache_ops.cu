// pa_reshape_and_cache and pa_copy_blocks for sm_100a.
//
// Cache write ("09. PagedAttention" (119-ai-studio), 해법; "Paged Attention"
// (velog @junegood), 작동 예시): each new token's K/V row of every KV head goes
// to the physical slot its block table assigns.  Copy-on-write ("KV Cache &
// PagedAttention" studynote, II; velog, 메모리 공유): a shared block is copied
// to a fresh block before a sharer writes into it.
//
// Both are pure data movement: 16-byte vector loads and stores, consecutive
// threads on consecutive 16-byte words of a row (coalesced reads and writes),
// grid-stride loops sized to a few waves of the 148 SMs.  Bad slots or block
// ids set err_flag and are skipped.
#include <algorithm>

#include "pa_common.cuh"

namespace pa {

__global__ void __launch_bounds__(256)
reshape_and_cache_kernel(const uint4* __restrict__ key, const uint4* __restrict__ value,
                         uint4* __restrict__ key_cache, uint4* __restrict__ value_cache,
                         const int64_t* __restrict__ slots, int64_t total, int row_vecs, int Hkv,
                         int bs, int64_t num_slots, int32_t* err) {
    // launched as a programmatic dependent of the kernel before it (e.g. the
    // previous step's decode, which may still read the cache): its blocks may
    // be resident early, but nothing is touched before that kernel completes
    grid_dependency_wait();
    // a decode launched after this kernel may be scheduled now; it waits on
    // the device for this grid's writes before it reads the cache
    launch_dependents();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t row = i / row_vecs;           // (token, head)
        const int c = (int)(i - row * row_vecs);
        const int64_t t = row / Hkv;
        const int h = (int)(row - t * Hkv);
        const int64_t s = __ldg(slots + t);
        if (s < 0) continue;                        // padding token
        if (s >= num_slots) {
            if (h == 0 && c == 0) set_err(err, PA_DEV_BAD_SLOT);
            continue;
        }
        const int64_t b = s / bs, o = s - b * bs;
        const int64_t dst = ((b * Hkv + h) * bs + o) * row_vecs + c;
        key_cache[dst] = __ldg(key + i);
        value_cache[dst] = __ldg(value + i);
    }
}

__global__ void __launch_bounds__(256)
copy_blocks_kernel(uint4* __restrict__ key_cache, uint4* __restrict__ value_cache,
                   const int64_t* __restrict__ pairs, int num_pairs, int64_t block_vecs,
                   int64_t num_blocks, int32_t* err) {
    uint4* cache = blockIdx.z ? value_cache : key_cache;
    for (int p = blockIdx.y; p < num_pairs; p += gridDim.y) {
        const int64_t src = __ldg(pairs + 2 * p), dst = __ldg(pairs + 2 * p + 1);
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) set_err(err, PA_DEV_BAD_PAIR);
            continue;
        }
        const uint4* s = cache + src * block_vecs;
        uint4* d = cache + dst * block_vecs;
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < block_vecs;
             i += (int64_t)gridDim.x * blockDim.x)
            d[i] = s[i];
    }
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

bool supported_shape(int head_dim, int block_size) {
    return (head_dim == 64 || head_dim == 128) &&
           (block_size == 8 || block_size == 16 || block_size == 32 || block_size == 64 ||
            block_size == 128);
}

int num_sms() {
    static int sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < 64) {
        if (!sms[dev]) cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
        return sms[dev] ? sms[dev] : 148;
    }
    return 148;
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" {

int pa_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                         const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                         int32_t* err_flag, void* stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0) return PA_ERR_INVALID;
    if (dtype != PA_F32 && dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_INVALID;
    if (!supported_shape(head_dim, block_size)) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_INVALID;
    if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
        return PA_ERR_INVALID;
    const int row_vecs = head_dim * (int)dtype_size(dtype) / 16;
    const int64_t total = (int64_t)num_tokens * num_kv_heads * row_vecs;
    const int64_t blocks = std::min<int64_t>((total + 255) / 256, (int64_t)num_sms() * 16);
    // programmatic dependent launch: the grid's launch overlaps the tail of
    // the kernel before it; the kernel waits (griddepcontrol.wait) for that
    // kernel to complete before its first global access
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = (cudaStream_t)stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(
        &cfg, reshape_and_cache_kernel, static_cast<const uint4*>(key),
        static_cast<const uint4*>(value), static_cast<uint4*>(key_cache),
        static_cast<uint4*>(value_cache), slot_mapping, total, row_vecs, num_kv_heads, block_size,
        (int64_t)num_blocks * block_size, err_flag);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int pa_copy_blocks(void* key_cache, void* value_cache, const int64_t* block_pairs, int num_pairs,
                   int num_kv_heads, int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                   int32_t* err_flag, void* stream) {
    if (num_pairs < 0 || num_kv_heads <= 0 || num_blocks <= 0) return PA_ERR_INVALID;
    if (dtype != PA_F32 && dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_INVALID;
    if (!supported_shape(head_dim, block_size)) return PA_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PA_OK;
    if (!key_cache || !value_cache || !block_pairs) return PA_ERR_INVALID;
    if (!aligned16(key_cache) || !aligned16(value_cache)) return PA_ERR_INVALID;
    const int64_t block_vecs =
        (int64_t)num_kv_heads * block_size * head_dim * (int64_t)dtype_size(dtype) / 16;
    const int64_t bx = std::min<int64_t>((block_vecs + 255) / 256, 64);
    const int by = std::min(num_pairs, 65535);
    dim3 grid((unsigned)bx, (unsigned)by, 2);
    copy_blocks_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(
        static_cast<uint4*>(key_cache), static_cast<uint4*>(value_cache), block_pairs, num_pairs,
        block_vecs, num_blocks, err_flag);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // extern "C"
