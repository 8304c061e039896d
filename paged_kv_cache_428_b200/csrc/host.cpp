// host.cpp -- host-only helpers of the C ABI: status text, version, KV-size closed form,
// and validation of host copies of block tables / slot ids.
#include <cstddef>
#include <cstdint>

#include "pa.h"

extern "C" {

const char *pa_status_str(int status)
{
    switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported shape (head_dim 64/128, block_size 16/32/64, group 1/2/4/8)";
    case PA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case PA_ERR_OOM: return "out of KV blocks";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_NOT_FOUND: return "unknown sequence id";
    default: return "unknown status";
    }
}

int pa_version(void) { return 100; }   // 0.1.0

// 2 (K and V) x layers x KV heads x head dim x bytes per element.
size_t pa_kv_bytes_per_token(int layers, int h_kv, int head_dim, int elem_bytes)
{
    if (layers < 0 || h_kv < 0 || head_dim < 0 || elem_bytes < 0) return 0;
    return 2u * (size_t)layers * (size_t)h_kv * (size_t)head_dim * (size_t)elem_bytes;
}

size_t pa_kv_capacity_tokens(size_t budget_bytes, int layers, int h_kv, int head_dim, int elem_bytes)
{
    const size_t per_token = pa_kv_bytes_per_token(layers, h_kv, head_dim, elem_bytes);
    return per_token ? budget_bytes / per_token : 0;
}

int pa_validate_block_tables(const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                             int num_seqs, int block_size, int num_blocks)
{
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || num_blocks <= 0) return PA_ERR_INVALID_ARG;
    if (num_seqs > 0 && (!block_tables || !context_lens)) return PA_ERR_INVALID_ARG;
    for (int s = 0; s < num_seqs; ++s) {
        const int ctx = context_lens[s];
        if (ctx < 0) return PA_ERR_INVALID_ARG;
        const long long used = ((long long)ctx + block_size - 1) / block_size;
        if (used > max_blocks_per_seq) return PA_ERR_INVALID_ARG;
        for (long long i = 0; i < used; ++i) {
            const int32_t b = block_tables[(size_t)s * max_blocks_per_seq + i];
            if (b < 0 || b >= num_blocks) return PA_ERR_INVALID_ARG;
        }
    }
    return PA_OK;
}

int pa_validate_slots(const int64_t *slot_mapping, int num_tokens, int block_size, int num_blocks)
{
    if (num_tokens < 0 || block_size <= 0 || num_blocks <= 0) return PA_ERR_INVALID_ARG;
    if (num_tokens > 0 && !slot_mapping) return PA_ERR_INVALID_ARG;
    const long long limit = (long long)num_blocks * block_size;
    for (int t = 0; t < num_tokens; ++t)
        if (slot_mapping[t] >= limit) return PA_ERR_INVALID_ARG;   // negative = padding, allowed
    return PA_OK;
}

}  // extern "C"
