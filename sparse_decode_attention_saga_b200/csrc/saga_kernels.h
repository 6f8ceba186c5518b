// Host-side launch interface of the kernels (internal to libsaga.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <utility>

#include "saga_params.h"

namespace saga {

// Launches `kern` after the previous kernel of the stream with programmatic
// stream serialization: its CTAs may be scheduled while that kernel drains,
// and the kernel calls pdl_wait() before it reads anything the previous one
// wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Makes kernel `fn` launchable with `bytes` of dynamic shared memory on the
// current device: above the 48 KB default the limit is raised, to the
// largest value asked for so far (never lowered).  CUDA keeps function
// attributes per device, so the limit is remembered per (kernel, device) (a
// process that drives several GPUs sets it on each before the kernel's
// first launch there).
cudaError_t allow_dynamic_smem(const void* fn, int bytes);
template <typename... KArgs>
cudaError_t allow_dynamic_smem(void (*kern)(KArgs...), int bytes) {
    return allow_dynamic_smem(reinterpret_cast<const void*>(kern), bytes);
}

// Streaming query-key kernel over the K cache (TMA pipeline + mma).
enum StreamMode : int {
    kStreamLogits = 0,  // write s = q.k/sqrt(d) to logits [b,hq,l]
    kStreamSelect = 1,  // compare s >= tau and append kept (pos, s) to lists
};

struct StreamArgs {
    Geometry g;
    int C;       // grid size (CTAs), <= kMaxCtas and <= b * tiles
    int stages;  // pipeline depth
    const void* q;
    const float* thresh;
    float* logits;
    int2* list;  // kept (position, logit bits) pairs, per (row, slot, warp) segment
    int32_t* seg_cnt;
    float* seg_mall;
    uint32_t* err;
};

size_t stream_smem_bytes(int stages);
cudaError_t launch_qk_stream(int mode, const CUtensorMap& kmap, const StreamArgs& a,
                             cudaStream_t stream);

// Radix select of the N-th largest logit per row.
struct RadixArgs {
    const float* logits;  // [rows][l]
    long long rows;
    int l;
    int N;
    int chunks;  // CTAs per row
    uint32_t* hist;
    uint32_t* state;
    uint32_t* tickets;
    float* thresh;
    uint32_t* err;
    // Digits to find (3: the whole threshold; 2: stop after pass 1 and leave
    // the last digit to the candidate compaction, which reads `state`).
    int passes;
    // Optional (nullable): pass 1 also copies (position, logit bits) of every
    // logit whose key is at or above the lower edge of pass 0's bucket into
    // chunk c's part [c*per, c*per + per) of cand[row][0..l) (per =
    // radix_chunk_len, in no fixed order) and their number into
    // cand_cnt[row][c]; pass 2 then reads only those (chunk c's CTA its own
    // chunk's).  Null: pass 2 reads the whole row again.
    int2* cand;
    int32_t* cand_cnt;
};
cudaError_t launch_radix_select(const RadixArgs& a, cudaStream_t stream);
// CTAs per row for the radix passes (cost model over waves and per-CTA overhead).
int radix_chunks(long long rows, int l, int sms);
// Positions per chunk of a row cut into `chunks` (a multiple of 4).
SAGA_HD int radix_chunk_len(int l, int chunks) { return ((l + chunks - 1) / chunks + 3) & ~3; }
// Adds n to the library's launch counter (saga_launch_count).
void note_launches(int n);
cudaError_t launch_fill(float* p, long long n, float value, cudaStream_t stream);

// Compare + ordered compaction of one logits row per CTA.
struct SelectArgs {
    const float* logits;  // [rows][l]
    const float* thresh;  // [rows]
    long long rows;
    int l;
    int32_t* idx;  // [rows][l]  kept positions, ascending
    float* s;      // [rows][l]  their logits, same order
    int32_t* cnt;  // [rows]
    float* rowmax; // [rows]     largest logit of the row
    int keep_max;  // nothing passed: keep the row's maxima (1) or nothing (0)
    int wide;      // few rows: 16 logits per thread per sub-round instead of 4
    uint32_t* empty_rows;  // optional: counts the rows that kept their maxima
    uint32_t* err;         // sticky flag (debug builds: bounds checks)
};
cudaError_t launch_select_compact(const SelectArgs& a, cudaStream_t stream);

// The same compare and ordered compaction over the candidates of the radix
// passes (RadixArgs::cand: every logit at or above the lower edge of the
// threshold's first-digit bucket, so every kept one, and the row's largest),
// one CTA per row with the row's bitmap of kept positions in shared memory.
// With `state` (the radix state after the first two digits), the kernel
// also finds the threshold's last digit from the candidates and writes the
// thresholds (the radix passes then stop after two digits).
struct CandSelectArgs {
    const int2* cand;          // [rows][l]  (position, logit bits), chunk c at c*per
    const int32_t* cand_cnt;   // [rows][kRadixMaxChunks]
    int chunks;                // the radix passes' chunks per row
    const uint32_t* state;     // nullable [rows][2]: (22-bit prefix, rank) after two digits
    float* thresh;             // [rows]: in, or out with state
    long long rows;
    int l;
    int32_t* idx;   // [rows][l]  kept positions, ascending
    float* s;       // [rows][l]  their logits, same order
    int32_t* cnt;   // [rows]
    float* rowmax;  // [rows]     largest logit of the row
    uint32_t* empty_rows;  // optional: counts the rows that kept their maxima
    uint32_t* err;         // sticky flag (debug builds: bounds checks)
};
size_t cand_select_smem(int l);
cudaError_t launch_cand_select(const CandSelectArgs& a, cudaStream_t stream);

// Ascending kept positions of every row from the fused kernel's per-(slot,
// warp) lists: the lists' positions are set in a per-row bitmap, which is
// then compacted in position order.  Rows that kept nothing are skipped (the
// row merge's empty-set fallback writes their positions).
struct IndexArgs {
    Geometry g;
    int C;                   // grid of the fused kernel
    const int2* seg_list;    // (position, logit bits) pairs [rows][l_pad]
    const int32_t* seg_cnt;  // [rows][S_cap][WPK]
    uint32_t* bitmap;        // scratch [rows][ceil(l/32)]
    int32_t* idx;            // [rows][l] out
    uint32_t* err;           // sticky flag (debug builds: bounds checks)
};
cudaError_t launch_lists_to_index(const IndexArgs& a, cudaStream_t stream);

// Log-sum-exp merge of partial records, plus the empty-set fallback.
enum CombineMode : int {
    kCombineParts = 0,     // `parts` records per row (gathered contiguous lists)
    kCombineSlots = 1,     // slots_of_batch records per row (fused / dense kernels)
};
struct CombineArgs {
    Geometry g;
    int mode;
    int parts;
    int C;
    int recs_per_slot;  // kCombineSlots: 1 (gathered lists) or WPK (dense kernel)
    int chunks;        // CTAs per row (0 or 1: one CTA merges the row)
    int partial_slot;  // chunks > 1: record slot of chunk 0's partial (past the inputs)
    uint32_t* tickets; // chunks > 1: per-row tickets, zero on entry and left at zero
    int fallback;      // recompute logits from q/K for rows that kept nothing
    const void* q;
    const void* k;
    const void* v;
    const float* records;
    float* out;
    int32_t* sel_cnt;
    // Optional: [rows][l] kept positions; written here only for rows that
    // kept nothing (the empty-set fallback's positions at the row maximum)
    int32_t* sel_idx;
    // Optional, for a sequence shard: the row's merged but unnormalised
    // record (m, l, count, row max, o[dv]) goes to part[row] instead of out
    // (count 0: m = -inf, l = number of positions at the row max, o = the
    // sum of their value rows).
    float* part;
    // Optional: counts the rows that kept nothing and took the empty-set
    // fallback (one atomic add per such row; not for a shard's partials).
    uint32_t* empty_rows;
    // Optional, with the fused kernel's lists (C its grid): the per-(slot,
    // warp) maxima [rows][S_cap][WPK], so that the fallback recomputes only
    // the lists that hold the row maximum.
    const float* seg_mall;
};
// Gathered softmax-PV over kept lists -> partial records.
enum ListMode : int {
    kListContiguous = 0,  // idx [rows][l], cnt [rows], s from logits
    kListSegments = 1,    // per (slot, sub-warp) lists from the fused kernel
};
struct GatherArgs {
    Geometry g;
    int mode;
    int parts;      // CTAs per row (each takes an equal share of the row's entries)
    int part_major; // grid (rows, parts) instead of (parts, rows)
    int C;          // kListSegments: grid of the fused kernel
    int max_lists;  // lists per row at most (kListSegments: slots * WPK; else 1)
    const void* v;
    const int32_t* idx;       // kListContiguous: positions [rows][l]
    const int32_t* cnt;       // kListContiguous: counts [rows]
    const float* rowmax;      // kListContiguous: largest logit per row [rows]
    const float* list_s;      // kListContiguous: logits of the listed entries [rows][l]
    const int2* seg_list;     // kListSegments: (position, logit bits) pairs [rows][l_pad]
    const int32_t* seg_cnt;
    const float* seg_mall;
    float* records;
    // The last CTA of each row (per-row tickets, zero on entry and left at
    // zero) merges the row's `parts` records as cmb describes.
    uint32_t* tickets;
    CombineArgs cmb;
    uint32_t* err;  // sticky flag (debug builds: bounds checks)
};
size_t gather_smem_bytes(int max_lists);
cudaError_t launch_gather_pv(const GatherArgs& a, cudaStream_t stream);

// Dense flash-decoding kernel (K and V streamed) -> partial records.
struct DenseArgs {
    Geometry g;
    int C;
    int stages;
    // Key heads of g per key head of the cache (1, or h_v / h_k when more
    // than two value heads share a key head: g then has one key head per
    // value head, and key head kh of g loads the cache's key head
    // kh / k_group, so that each such head's query heads use one value head).
    int k_group;
    const void* q;
    float* records;
    uint32_t* err;
};
// Shapes the dense kernel handles: h_v <= 2 h_k, value heads aligned with
// the key-head groups (geometries with more value heads per key head go
// through the k_group form above).
bool dense_supported(const Geometry& g);
size_t dense_stage_bytes(const Geometry& g);
size_t dense_smem_bytes(const Geometry& g, int stages);
cudaError_t launch_dense(const CUtensorMap& kmap, const CUtensorMap& vmap, const DenseArgs& a,
                         cudaStream_t stream);

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream);

// Sequence shards: digit histograms of this shard's logits (summed across
// shards by the caller), the digit choice on the summed histograms, and the
// merge of the shards' partial records.
struct ShardHistArgs {
    const float* logits;    // [rows][l] this shard's logits
    long long rows;
    int l;
    int chunks;             // CTAs per row
    const uint32_t* state;  // [rows][2] (prefix, rank) of the earlier passes
    uint32_t* hist;         // [rows][kRadixBins] out (cleared first)
};
cudaError_t launch_shard_hist(int pass, const ShardHistArgs& a, cudaStream_t stream);
struct ShardDigitArgs {
    const uint32_t* hist;   // [rows][kRadixBins] summed over the shards
    long long rows;
    int N;
    uint32_t* state;        // [rows][2] in/out; rank 0: threshold known
    float* thresh;          // [rows] written once known
};
cudaError_t launch_shard_digit(int pass, const ShardDigitArgs& a, cudaStream_t stream);
struct MergeArgs {
    const float* parts;     // [R][rows][dv + kRecHeader]
    int R;
    long long rows;
    float* out;             // [rows][dv]
    int32_t* sel_cnt;       // [rows] or null
};
cudaError_t launch_merge_parts(int dv, const MergeArgs& a, cudaStream_t stream);

// Cache growth: new rows k_new [b,h_k,d], v_new [b,h_v,d] -> row `pos` of
// k [b,l_cap,h_k,d] and v [b,l_cap,h_v,d].
struct AppendArgs {
    int b, hk, hv, d, dv, l_cap, pos;  // d: key head dim, dv: value head dim
    const void* k_new;
    const void* v_new;
    void* k;
    void* v;
};
cudaError_t launch_cache_append(const AppendArgs& a, cudaStream_t stream);

}  // namespace saga
