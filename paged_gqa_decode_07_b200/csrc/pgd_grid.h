// pgd_grid.h -- how the decode entry points size their grid and weigh the
// work of a (sequence, KV head) unit in the kernel's work cut (host code).
#pragma once

#include <stdint.h>

#include <algorithm>

#include "pgd_decode.cuh"

namespace pgd {

// Fixed cost of one (sequence, KV head) unit in a CTA (descriptor, query
// rows, block-table fetch, first-tile latency, merge, output) expressed as the
// K/V bytes a CTA streams in the same time.  FP8 tiles take longer per byte
// (the consumers convert every element), so the same time is fewer bytes.
// The batch is cut by tiles + this many tile-equivalents per unit.
constexpr long long kUnitOverheadBytes = 48 * 1024;
constexpr long long kUnitOverheadBytesFp8 = 36 * 1024;

inline int32_t unit_cost_tiles(int head_dim, int block_size, bool fp8) {
    const long long tile_kv = 2LL * block_size * head_dim * (fp8 ? 1 : 2);
    const long long unit = fp8 ? kUnitOverheadBytesFp8 : kUnitOverheadBytes;
    return static_cast<int32_t>((unit + tile_kv - 1) / tile_kv);
}

// Automatic grid: one wave of resident CTAs (sms x occ), fewer for small
// batches (at least 4 stages of work per CTA, counting each unit's fixed
// cost, so that a batch of many short units still fills the wave).  With
// fewer (sequence, KV head) units than CTAs, units of equal length should
// split into whole pieces, one per CTA, not CTAs that hold the ends of two:
// a small batch takes the multiple of the unit count nearest that cap, and a
// full wave is rounded down to a multiple of it when that drops at most 1/8
// of the wave.
inline long long auto_grid(int sms, int occ, int32_t num_seqs, int32_t num_kv_heads,
                           int32_t max_blocks_per_seq, int32_t block_size,
                           int32_t max_context_len, int32_t unit_cost) {
    const long long units = static_cast<long long>(num_seqs) * num_kv_heads;
    const long long cap_tokens = static_cast<long long>(max_blocks_per_seq) * block_size;
    const long long max_ctx =
        max_context_len > 0 ? std::min<long long>(max_context_len, cap_tokens) : cap_tokens;
    const long long work_upper = units * ((max_ctx + block_size - 1) / block_size + unit_cost);
    const long long min_work = 4 * (kStageTokens / block_size);   // >= 4 stages per CTA
    const long long full = static_cast<long long>(sms) * occ;
    const long long cap = (work_upper + min_work - 1) / min_work;
    long long grid = std::min(full, cap);
    if (units > 0 && units < grid) {
        if (cap < full) {
            const long long pieces = std::max(1LL, (cap + units / 2) / units);
            grid = std::min(pieces, full / units) * units;
        } else if (grid % units <= grid / 8) {
            grid -= grid % units;
        }
    }
    return std::max(1LL, grid);
}

}  // namespace pgd
