// Launch plan and workspace layout of one ISD step, derived from the dims
// alone (no device data is read on the host, so every call is capturable).
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/isd.h"

namespace isd {

constexpr int kAttnKeyTile = 64;      // keys per pipeline stage
constexpr int kAttnRowsPerGroup = 16; // query rows handled by one 4-warp group
constexpr int kAttnMaxSplit = 2048;   // keys per split at most (bounds the key table)
constexpr int kStatsThreads = 256;
constexpr int kFinalizeThreads = 256;   // one CTA per row merges its statistics partials
constexpr int kAcceptThreads = 256;
// Vocabulary entries per accept CTA (2048 measured 19% faster for the accept
// kernel than 4096 at B=32, N=4, V=151936; the chunk totals of a request are
// scanned by one CTA, so V <= kAcceptThreads * kAcceptChunk).
constexpr int kAcceptChunk = 2048;
// accept CTAs resident per SM (launch bounds: 64 registers a thread)
constexpr int kAcceptMinBlocks = 4;
// SDAR block size limit (one warp per block row in the unmask kernel)
constexpr int kSdarMaxN = 16;
// Persistent kernels (attention, LM head) run one CTA per SM of the current
// device, at most kMaxSMs (a B200 has 148); the workspace is sized for
// kMaxSMs, and the split heuristics below aim at a B200-sized grid.
constexpr int kMaxSMs = 192;
constexpr int kPlanSMs = 148;
// row-statistics partials per logits row at most (the LM head's epilogue
// writes one per CTA plus two per left-over pair tile; merged by one warp)
constexpr int kMaxStatParts = 384;
// LM head: accumulator columns for Mh hidden rows (one block of <= 256
// columns, or two equal blocks), each a multiple of 16
inline int lm_cols(int Mh) {
    if (Mh <= 256) return (Mh + 15) / 16 * 16;
    return 2 * (((Mh + 1) / 2 + 15) / 16 * 16);
}
// floats of one CTA's tile-tail buffer: its 128 vocabulary rows x lm_cols
inline size_t lm_part_floats(int Mh) { return (size_t)128 * lm_cols(Mh); }

struct Plan {
    // derived dims
    int Q, H, M, grp, rows;  // rows = grp * Q query rows per (request, kv head)
    // attention
    int attn_rg;             // 16-row warp groups per CTA (1, 2 or 4)
    int attn_rgb;            // row-group blocks per (request, kv head)
    int attn_split;          // keys per split (multiple of kAttnKeyTile)
    int attn_max_splits;     // splits for the longest possible request
    size_t attn_part_stride; // bytes of one split's partial
    // tensor-core attention (D = 128, pages dividing 128 keys, <= 64 rows):
    // rows padded to the MMA N (16, 32 or 64), 0 when the shape does not fit
    int attn_tc_rows;
    int attn_tc_part_stride; // floats of one partial (per CTA and slot)
    // statistics / accept
    int stats_chunks, stats_chunk_len;
    int acc_chunks;
    // R-ISD LoRA
    int lora_rows, lora_ksplit;
    // LM-head row-statistics partials per row: room for one per CTA and two
    // per left-over pair tile (the launch decides how many are used)
    int lm_stat_parts;
    // workspace offsets (bytes)
    size_t off_attn_part, off_attn_ticket, off_hidden, off_hidden_lora, off_lora_t,
        off_stats_part, off_stats_ticket, off_acc_part, off_acc_ticket, off_lora_part,
        off_lm_stats, off_lm_tail, total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// SMs of the current device, capped at kMaxSMs (cached per device).  The one
// place the persistent kernels take their grid size from.
int persistent_grid();

// Returns false if the dims are invalid.  block_q: query rows per request;
// 0 means the ISD block of 2N - 1 slots (an SDAR block has N).
inline bool make_plan(const isd_dims* d, Plan* p, int block_q = 0) {
    if (!d || d->B < 1 || d->N < 1 || d->Hq < 1 || d->Hkv < 1 || d->D < 1 || d->V < 1 ||
        d->page_size < 1 || d->num_pages < 1 || d->max_pages_per_req < 1 || d->lora_rank < 0 ||
        d->Hq % d->Hkv != 0 ||
        (d->proposal_mode != ISD_PROPOSE_ARGMAX && d->proposal_mode != ISD_PROPOSE_SAMPLE))
        return false;
    p->Q = block_q > 0 ? block_q : 2 * d->N - 1;
    p->H = d->Hq * d->D;
    p->M = d->B * p->Q;
    p->grp = d->Hq / d->Hkv;
    p->rows = p->grp * p->Q;
    p->attn_rg = p->rows <= 16 ? 1 : (p->rows <= 32 ? 2 : 4);
    const int rows_per_cta = kAttnRowsPerGroup * p->attn_rg;
    p->attn_rgb = (p->rows + rows_per_cta - 1) / rows_per_cta;
    const long long max_ctx = (long long)d->max_pages_per_req * d->page_size;
    // Aim for about 3 waves of 2 CTAs per SM over the expected keys (half
    // the longest context per request on average).
    long long est = (long long)d->B * d->Hkv * p->attn_rgb * (max_ctx / 2 + 1);
    long long split = est / (kPlanSMs * 2 * 3);
    if (split < 256) split = 256;
    if (split > kAttnMaxSplit) split = kAttnMaxSplit;
    split = (split + kAttnKeyTile - 1) / kAttnKeyTile * kAttnKeyTile;
    p->attn_split = (int)split;
    p->attn_max_splits = (int)((max_ctx + split - 1) / split);
    if (p->attn_max_splits < 1) p->attn_max_splits = 1;
    p->attn_part_stride = align_up((size_t)rows_per_cta * d->D * 4 + (size_t)rows_per_cta * 8, 256);
    const int P = d->page_size;
    const bool tc_pages = P == 8 || P == 16 || P == 32 || P == 64 || P == 128;
    p->attn_tc_rows = 0;
    if (d->D == 128 && tc_pages && p->rows <= 64)
        p->attn_tc_rows = p->rows <= 16 ? 16 : (p->rows <= 32 ? 32 : 64);
    p->attn_tc_part_stride = 2 * p->attn_tc_rows + 128 * p->attn_tc_rows;
    // row statistics: enough CTAs to fill the GPU, chunks of >= 2048 entries
    int target = (kPlanSMs * 8 + p->M - 1) / p->M;
    int max_chunks = (d->V + 2047) / 2048;
    p->stats_chunks = target < 1 ? 1 : (target > max_chunks ? max_chunks : target);
    if (p->stats_chunks < 1) p->stats_chunks = 1;
    p->stats_chunk_len = (int)align_up((size_t)((d->V + p->stats_chunks - 1) / p->stats_chunks), 4);
    p->acc_chunks = (d->V + kAcceptChunk - 1) / kAcceptChunk;
    p->lora_rows = d->B * (d->N - 1);
    p->lora_ksplit = 1;
    if (d->lora_rank > 0) {
        // split the long K = H reduction of h.A so that about 100 CTAs work on it
        const int tiles = ((p->lora_rows + 63) / 64) * ((d->lora_rank + 63) / 64);
        int ks = (100 + tiles - 1) / tiles;
        const int kiters = p->H / 32;
        if (ks > kiters) ks = kiters;
        if (ks < 1) ks = 1;
        p->lora_ksplit = ks;
    }
    // workspace
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    const size_t n_units = (size_t)d->B * d->Hkv * p->attn_rgb;
    // split partials of the general kernel, or two partials per persistent
    // CTA of the tensor-core kernel: whichever is larger
    size_t part_bytes = n_units * p->attn_max_splits * p->attn_part_stride;
    const size_t tc_bytes = (size_t)kMaxSMs * 2 * p->attn_tc_part_stride * 4;
    if (tc_bytes > part_bytes) part_bytes = tc_bytes;
    p->off_attn_part = take(part_bytes);
    p->off_attn_ticket = take(n_units * 4);
    p->off_hidden = take((size_t)p->M * p->H * 2);
    p->off_hidden_lora = take(d->lora_rank ? (size_t)p->M * p->H * 2 : 0);
    p->off_lora_t = take(d->lora_rank ? (size_t)p->M * d->lora_rank * 2 : 0);
    p->off_stats_part = take((size_t)p->M * p->stats_chunks * 16);
    p->off_stats_ticket = take((size_t)p->M * 4);
    p->off_acc_part = take((size_t)d->B * (d->N + 1) * p->acc_chunks * 4);
    p->off_acc_ticket = take((size_t)d->B * 2 * 4 + 4);  // tickets, decided states, decided count
    p->off_lora_part = take(d->lora_rank ? (size_t)p->lora_ksplit * p->lora_rows * d->lora_rank * 4 : 0);
    p->lm_stat_parts = kMaxStatParts;
    p->off_lm_stats = take((size_t)p->M * p->lm_stat_parts * 16);
    // LM head: one tile-tail accumulator buffer and one flag per CTA
    p->off_lm_tail = take((size_t)kMaxSMs * lm_part_floats(p->M) * 4 + (size_t)kMaxSMs * 4);
    p->total = off;
    return true;
}

}  // namespace isd
