// Cache-side kernels: KV append (reshape_and_cache), block copy (copy_blocks)
// and block swap between a device pool and a page-locked host pool (swap_blocks).
//
// Layout ("LLM 推理引擎内部原理" §2.4): cache[num_blocks, block_size, Hkv, D].
// One token's K (or V) for all heads is one contiguous row of Hkv*D elements
// at (slot / block_size, slot % block_size), so the append is a row copy, and a
// physical block is one contiguous span of block_size*Hkv*D elements, so the
// block copy is a span copy. Both move 16-byte vectors, several in flight per
// thread, with non-allocating loads of the read-once source.
#include <cmath>

#include "common.cuh"

namespace pkv {
namespace {

__device__ __forceinline__ int4 ld_stream(const int4* p) {
    int4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.s32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// grid.x = token, grid.y = 0 (K) / 1 (V). Each CTA copies one row of
// row_vecs 16-byte vectors.
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const int4* __restrict__ k, const int4* __restrict__ v, int4* __restrict__ k_cache,
    int4* __restrict__ v_cache, const int64_t* __restrict__ slot_mapping, int row_vecs,
    int64_t num_slots, int* err) {
    const int t = blockIdx.x;
    const int64_t slot = slot_mapping[t];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (threadIdx.x == 0) flag_error(err, PKV_ERR_DEVICE_BOUNDS);
        return;
    }
    const int4* src = (blockIdx.y == 0 ? k : v) + (int64_t)t * row_vecs;
    int4* dst = (blockIdx.y == 0 ? k_cache : v_cache) + slot * row_vecs;
    int i = threadIdx.x;
    for (; i + 3 * 256 < row_vecs; i += 4 * 256) {
        int4 a = ld_stream(src + i), b = ld_stream(src + i + 256);
        int4 c = ld_stream(src + i + 512), d = ld_stream(src + i + 768);
        dst[i] = a;
        dst[i + 256] = b;
        dst[i + 512] = c;
        dst[i + 768] = d;
    }
    for (; i < row_vecs; i += 256) dst[i] = ld_stream(src + i);
}

// FP8 append: grid.x = token, grid.y = 0 (K) / 1 (V). Each thread turns 16
// input elements (bf16 or fp32) into one 16-byte vector of e4m3 codes:
// code = e4m3(x * inv_scale) with round to nearest even and saturation.
template <typename TIn>
__global__ void __launch_bounds__(256) reshape_and_cache_fp8_kernel(
    const TIn* __restrict__ k, const TIn* __restrict__ v, uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
    float k_inv, float v_inv, const int64_t* __restrict__ slot_mapping, int row_elems, int64_t num_slots, int* err) {
    const int t = blockIdx.x;
    const int64_t slot = slot_mapping[t];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (threadIdx.x == 0) flag_error(err, PKV_ERR_DEVICE_BOUNDS);
        return;
    }
    const bool is_k = blockIdx.y == 0;
    const TIn* src = (is_k ? k : v) + (int64_t)t * row_elems;
    uint4* dst = (is_k ? k_cache : v_cache) + slot * (row_elems / 16);
    const float inv = is_k ? k_inv : v_inv;
    for (int c = threadIdx.x; c < row_elems / 16; c += 256) {
        float f[16];
        if constexpr (sizeof(TIn) == 4) {
            const float4* s4 = reinterpret_cast<const float4*>(src + c * 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 x = s4[i];
                f[4 * i] = x.x; f[4 * i + 1] = x.y; f[4 * i + 2] = x.z; f[4 * i + 3] = x.w;
            }
        } else {
            const uint4* s4 = reinterpret_cast<const uint4*>(src + c * 16);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const uint4 x = s4[i];
                f[8 * i] = bf16lo(x.x); f[8 * i + 1] = bf16hi(x.x); f[8 * i + 2] = bf16lo(x.y);
                f[8 * i + 3] = bf16hi(x.y); f[8 * i + 4] = bf16lo(x.z); f[8 * i + 5] = bf16hi(x.z);
                f[8 * i + 6] = bf16lo(x.w); f[8 * i + 7] = bf16hi(x.w);
            }
        }
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = float2_to_e4m3x2(__fmul_rn(f[4 * i], inv), __fmul_rn(f[4 * i + 1], inv));
            const uint32_t hi = float2_to_e4m3x2(__fmul_rn(f[4 * i + 2], inv), __fmul_rn(f[4 * i + 3], inv));
            w[i] = lo | (hi << 16);
        }
        dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// grid.x = chunk of the block span (kChunkVecs vectors), grid.y = pair,
// grid.z = 0 (K) / 1 (V). Copies block src_ids[y] of the source pool to block
// dst_ids[y] of the destination pool (the same pool for copy-on-write copies).
// A source in device memory is read through the non-coherent streaming path; a
// source in mapped host memory (swap-in) with plain loads, several 16-byte
// vectors in flight per thread to cover the host link's latency.
constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;
constexpr int kChunkVecs = kCopyThreads * kCopyUnroll;

template <bool kDeviceSrc>
__global__ void __launch_bounds__(kCopyThreads) block_copy_kernel(
    const int4* __restrict__ src_k, const int4* __restrict__ src_v, int4* __restrict__ dst_k,
    int4* __restrict__ dst_v, const int64_t* __restrict__ src_ids, const int64_t* __restrict__ dst_ids,
    int64_t block_vecs, int64_t src_blocks, int64_t dst_blocks, int* err) {
    const int64_t s = src_ids[blockIdx.y], d = dst_ids[blockIdx.y];
    if (s < 0 || s >= src_blocks || d < 0 || d >= dst_blocks) {
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0) flag_error(err, PKV_ERR_DEVICE_BOUNDS);
        return;
    }
    const int4* src = (blockIdx.z == 0 ? src_k : src_v) + s * block_vecs;
    int4* dst = (blockIdx.z == 0 ? dst_k : dst_v) + d * block_vecs;
    const int64_t base = (int64_t)blockIdx.x * kChunkVecs + threadIdx.x;
    int4 r[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const int64_t i = base + u * kCopyThreads;
        if (i < block_vecs) r[u] = kDeviceSrc ? ld_stream(src + i) : src[i];
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const int64_t i = base + u * kCopyThreads;
        if (i < block_vecs) dst[i] = r[u];
    }
}

// A pointer the kernels can use for p: device (or managed) memory as is, page-
// locked host memory through its mapped device address. Pageable host memory
// and unknown pointers give nullptr. *host tells which.
void* device_view(const void* p, bool* host) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return nullptr;
    }
    *host = a.type == cudaMemoryTypeHost;
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return const_cast<void*>(p);
    if (a.type == cudaMemoryTypeHost && a.devicePointer) {
        // the mapped address of p itself (p may point inside the allocation)
        const char* base_h = static_cast<const char*>(a.hostPointer);
        return static_cast<char*>(a.devicePointer) + (static_cast<const char*>(p) - base_h);
    }
    return nullptr;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elt_bytes(pkv_dtype t) { return t == PKV_F32 ? 4 : (t == PKV_BF16 ? 2 : (t == PKV_FP8_E4M3 ? 1 : 0)); }

}  // namespace
}  // namespace pkv

extern "C" {

pkv_status pkv_reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                                 pkv_dtype dtype, const int64_t* slot_mapping, int num_tokens,
                                 int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                 void* stream) {
    using namespace pkv;
    const int eb = elt_bytes(dtype);
    if (eb == 0 || num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0)
        return PKV_ERR_INVALID_ARG;
    const int64_t row_bytes = (int64_t)num_kv_heads * head_dim * eb;
    if (row_bytes % 16 != 0 || row_bytes / 16 > INT32_MAX) return PKV_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PKV_OK;
    if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
        return PKV_ERR_INVALID_ARG;
    int* err = device_error_word();
    if (!err) return PKV_ERR_CUDA;
    dim3 grid(num_tokens, 2);
    reshape_and_cache_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const int4*>(k), static_cast<const int4*>(v), static_cast<int4*>(k_cache),
        static_cast<int4*>(v_cache), slot_mapping, (int)(row_bytes / 16),
        (int64_t)num_blocks * block_size, err);
    return cuda_status(cudaGetLastError());
}

pkv_status pkv_reshape_and_cache_fp8(const void* k, const void* v, pkv_dtype in_dtype, void* k_cache, void* v_cache,
                                     float k_scale, float v_scale, const int64_t* slot_mapping, int num_tokens,
                                     int num_kv_heads, int head_dim, int block_size, int num_blocks, void* stream) {
    using namespace pkv;
    if ((in_dtype != PKV_F32 && in_dtype != PKV_BF16) || num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_blocks <= 0 || !(k_scale > 0.f) || !(v_scale > 0.f) || !std::isfinite(k_scale) ||
        !std::isfinite(v_scale))
        return PKV_ERR_INVALID_ARG;
    const int64_t row = (int64_t)num_kv_heads * head_dim;
    if (row % 16 != 0 || row > INT32_MAX) return PKV_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PKV_OK;
    if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache)) return PKV_ERR_INVALID_ARG;
    int* err = device_error_word();
    if (!err) return PKV_ERR_CUDA;
    const float k_inv = 1.0f / k_scale, v_inv = 1.0f / v_scale;
    dim3 grid(num_tokens, 2);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (in_dtype == PKV_F32)
        reshape_and_cache_fp8_kernel<float><<<grid, 256, 0, st>>>(
            static_cast<const float*>(k), static_cast<const float*>(v), static_cast<uint4*>(k_cache),
            static_cast<uint4*>(v_cache), k_inv, v_inv, slot_mapping, (int)row, (int64_t)num_blocks * block_size, err);
    else
        reshape_and_cache_fp8_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
            static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), static_cast<uint4*>(k_cache),
            static_cast<uint4*>(v_cache), k_inv, v_inv, slot_mapping, (int)row, (int64_t)num_blocks * block_size, err);
    return cuda_status(cudaGetLastError());
}

pkv_status pkv_copy_blocks(void* k_cache, void* v_cache, pkv_dtype dtype,
                           const int64_t* src_block_ids, const int64_t* dst_block_ids, int num_pairs,
                           int block_size, int num_kv_heads, int head_dim, int num_blocks,
                           void* stream) {
    using namespace pkv;
    const int eb = elt_bytes(dtype);
    if (eb == 0 || num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0 || num_pairs > 65535)
        return PKV_ERR_INVALID_ARG;
    const int64_t block_bytes = (int64_t)block_size * num_kv_heads * head_dim * eb;
    if (block_bytes % 16 != 0) return PKV_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PKV_OK;
    if (!k_cache || !v_cache || !src_block_ids || !dst_block_ids) return PKV_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache)) return PKV_ERR_INVALID_ARG;
    int* err = device_error_word();
    if (!err) return PKV_ERR_CUDA;
    const int64_t block_vecs = block_bytes / 16;
    const int64_t chunks = (block_vecs + kChunkVecs - 1) / kChunkVecs;
    if (chunks > INT32_MAX) return PKV_ERR_UNSUPPORTED;
    dim3 grid((unsigned)chunks, num_pairs, 2);
    block_copy_kernel<true><<<grid, kCopyThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const int4*>(k_cache), static_cast<const int4*>(v_cache), static_cast<int4*>(k_cache),
        static_cast<int4*>(v_cache), src_block_ids, dst_block_ids, block_vecs, num_blocks, num_blocks, err);
    return cuda_status(cudaGetLastError());
}

pkv_status pkv_swap_blocks(const void* src_k_cache, const void* src_v_cache, int src_num_blocks, void* dst_k_cache,
                           void* dst_v_cache, int dst_num_blocks, pkv_dtype dtype, const int64_t* src_block_ids,
                           const int64_t* dst_block_ids, int num_pairs, int block_size, int num_kv_heads,
                           int head_dim, void* stream) {
    using namespace pkv;
    const int eb = elt_bytes(dtype);
    if (eb == 0 || num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        src_num_blocks <= 0 || dst_num_blocks <= 0 || num_pairs > 65535)
        return PKV_ERR_INVALID_ARG;
    const int64_t block_bytes = (int64_t)block_size * num_kv_heads * head_dim * eb;
    if (block_bytes % 16 != 0) return PKV_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PKV_OK;
    if (!src_k_cache || !src_v_cache || !dst_k_cache || !dst_v_cache || !src_block_ids || !dst_block_ids)
        return PKV_ERR_INVALID_ARG;
    if (!aligned16(src_k_cache) || !aligned16(src_v_cache) || !aligned16(dst_k_cache) || !aligned16(dst_v_cache))
        return PKV_ERR_INVALID_ARG;
    bool hk, hv, dk_host, dv_host, hs, hd;
    const void* sk = device_view(src_k_cache, &hk);
    const void* sv = device_view(src_v_cache, &hv);
    void* dk = device_view(dst_k_cache, &dk_host);
    void* dv = device_view(dst_v_cache, &dv_host);
    const void* ids_s = device_view(src_block_ids, &hs);
    const void* ids_d = device_view(dst_block_ids, &hd);
    if (!sk || !sv || !dk || !dv || !ids_s || !ids_d || hk != hv || dk_host != dv_host) return PKV_ERR_INVALID_ARG;
    int* err = device_error_word();
    if (!err) return PKV_ERR_CUDA;
    const int64_t block_vecs = block_bytes / 16;
    const int64_t chunks = (block_vecs + kChunkVecs - 1) / kChunkVecs;
    if (chunks > INT32_MAX) return PKV_ERR_UNSUPPORTED;
    dim3 grid((unsigned)chunks, num_pairs, 2);
    auto st = static_cast<cudaStream_t>(stream);
    auto kern = hk ? block_copy_kernel<false> : block_copy_kernel<true>;
    kern<<<grid, kCopyThreads, 0, st>>>(static_cast<const int4*>(sk), static_cast<const int4*>(sv),
                                        static_cast<int4*>(dk), static_cast<int4*>(dv),
                                        static_cast<const int64_t*>(ids_s), static_cast<const int64_t*>(ids_d),
                                        block_vecs, src_num_blocks, dst_num_blocks, err);
    return cuda_status(cudaGetLastError());
}

}  // extern "C"
