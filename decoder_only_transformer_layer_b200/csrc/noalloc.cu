// Decode attention that allocates no device memory.
//
// gqa_decode_attn keeps its scratch (per-split partial results and merge counters) in
// buffers it allocates on first use. Some callers cannot let a library allocate:
// a host program whose device memory is entirely reserved up front by its own pool
// allocator (a stray cudaMalloc then fails, or fragments the pool), a latency-bound
// serving loop that cannot absorb the device-wide synchronisation a cudaMalloc or
// cudaFree may cause, or a plugin host that forbids allocation after start-up. This
// file gives them the same kernel with its scratch in a fixed array that is part of
// the library image: it exists on every device that loads the library and lives until
// the process exits.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <string>

#include "../../include/dec_api.h"
#include "kernels.h"

namespace {

// Capacity of the fixed scratch: merge counters first, then split partials.
constexpr size_t kCounterCap = 16384;                // (sequence, kv head) pairs
constexpr size_t kPartialCap = (size_t)1 << 20;      // partial floats (4 MiB)
constexpr size_t kCounterBytes = kCounterCap * sizeof(int);
constexpr size_t kScratchBytes = kCounterBytes + kPartialCap * sizeof(float);

static __device__ __align__(256) unsigned char noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void* g_addr[256];  // host-usable address of noalloc_scratch on each device, set on first use

dec_status bad(dec_status s, const std::string& why) {
    dec::set_last_error(why);
    return s;
}

}  // namespace

extern "C" dec_status gqa_decode_attn_noalloc(const void* q, const void* k_new, const void* v_new, void* k_pool,
                                              void* v_pool, const int32_t* block_table, int32_t max_pages,
                                              const int32_t* pos, int32_t B, int32_t nq, int32_t nkv, int32_t d,
                                              int32_t page_size, float scale, int32_t fused_rope, float rope_base,
                                              void* out, dec_stream_t stream) {
    dec::set_last_error("");
    if (!q || !k_pool || !v_pool || !block_table || !pos || !out) return bad(DEC_ERR_INVALID_ARG, "NULL pointer");
    if ((k_new == nullptr) != (v_new == nullptr)) return bad(DEC_ERR_INVALID_ARG, "k_new and v_new: both or neither");
    if (B <= 0 || nq <= 0 || nkv <= 0 || nq % nkv != 0 || max_pages <= 0)
        return bad(DEC_ERR_INVALID_ARG, "bad B / heads / max_pages");
    if (nq / nkv > 16) return bad(DEC_ERR_UNSUPPORTED, "more than 16 q heads per kv head");
    if (d != 64 && d != 128) return bad(DEC_ERR_UNSUPPORTED, "d must be 64 or 128");
    if (page_size != 16) return bad(DEC_ERR_UNSUPPORTED, "page_size must be 16");

    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return bad(DEC_ERR_CUDA, "no current device");
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // Same split choice as gqa_decode_attn, so both calls sum in the same order.
    const int splits = dec::attn_decode_splits(B, nkv, max_pages * 16, sms, false);
    const size_t counters = (size_t)B * nkv;
    const size_t partials = splits > 1 ? (size_t)B * nq * splits * (d + 2) : 0;
    if (counters > kCounterCap)
        return bad(DEC_ERR_UNSUPPORTED, "B * n_kv_heads exceeds the fixed scratch (16384 pairs)");
    if (partials > kPartialCap)
        return bad(DEC_ERR_UNSUPPORTED, "split partials exceed the fixed scratch (1048576 floats)");

    void* base = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_addr[dev]) {
            // first call on this device: resolve the device address of the array
            cudaError_t e = cudaGetSymbolAddress(&g_addr[dev], noalloc_scratch);
            if (e != cudaSuccess) {
                g_addr[dev] = nullptr;
                return bad(DEC_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
            }
        }
        base = g_addr[dev];
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int* cnt = static_cast<int*>(base);
    float* part = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + kCounterBytes);
    // The merge counters must start at zero; the array keeps whatever the last call left.
    cudaError_t e = cudaMemsetAsync(cnt, 0, counters * sizeof(int), st);
    if (e != cudaSuccess) return bad(DEC_ERR_CUDA, std::string("cudaMemsetAsync: ") + cudaGetErrorString(e));

    dec::AttnDecodeArgs a{};
    a.q_bf = static_cast<const uint16_t*>(q);
    a.k_new = static_cast<const uint16_t*>(k_new);
    a.v_new = static_cast<const uint16_t*>(v_new);
    a.eps = 1e-6f;
    a.rope = fused_rope;
    a.rope_base = rope_base;
    a.k_pool = static_cast<uint16_t*>(k_pool);
    a.v_pool = static_cast<uint16_t*>(v_pool);
    a.block_table = block_table;
    a.max_pages = max_pages;
    a.pos = pos;
    a.B = B;
    a.nq = nq;
    a.nkv = nkv;
    a.d = d;
    a.scale = scale;
    a.splits = splits;
    a.part = part;
    a.counters = cnt;
    a.out = static_cast<uint16_t*>(out);
    a.err = nullptr;
    e = dec::attn_decode_launch(a, st, false);
    if (e != cudaSuccess) return bad(DEC_ERR_CUDA, std::string("launch: ") + cudaGetErrorString(e));
    return DEC_OK;
}
