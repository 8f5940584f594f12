// Tile scheduler: splits the decode work of a batch into `num_parts` contiguous
// ranges of nearly equal cost, one per two-SM cluster of the split-KV kernel.
//
// "FlashMLA" usage page (deepep.org): get_mla_metadata analyses the sequence
// lengths once per decoding step and returns tile_scheduler_metadata and
// num_splits, reused by every layer; its Tile Scheduler "distributes work across
// GPU resources" and balances variable-length sequences ("optimized for
// variable-length sequence serving", sourcepulse summary).  The pages do not
// print the algorithm or the metadata format; this one is our own.
//
// Work units.  A "virtual batch" vb = b * row_groups + g is request b restricted
// to query rows [128 g, 128 g + 128) of its s_q * h_q rows.  Its cost is its
// page count ceil(L_b / 64) plus kFixedCost pages of per-chunk overhead (Q load,
// epilogue).  Walking the virtual batches in order, each partition takes
// budget T = ceil(W / num_parts) + kFixedCost of cost (the extra kFixedCost pays
// for the chunk a split adds, so the budgets cover the total); a virtual batch
// that does not fit whole is cut at a page boundary and continues in the next
// partition (a split).  The last partition takes whatever remains.
//
// Output:
//   md[p * 8 + 0..4] = begin_vb, begin_blk, end_vb, end_blk, begin_split
//     partition p covers the positions (vb, blk) with
//     (begin_vb, begin_blk) <= (vb, blk) < (end_vb, end_blk) in lexicographic
//     order; a virtual batch with no pages is the single position (vb, 0).
//     begin_split is the split index of partition p's first chunk within
//     begin_vb (later chunks of the partition start their virtual batch, index 0).
//   num_splits[vb] = sum of split counts of virtual batches before vb
//     (num_splits[NV] = total), so vb has num_splits[vb+1] - num_splits[vb] splits
//     and its k-th split result goes to workspace slot num_splits[vb] + k.
#pragma once

#include <cstdint>

#ifdef __CUDACC__
#define MLA_HD __host__ __device__
#else
#define MLA_HD
#endif

namespace mla {

constexpr int kPage = 64;
constexpr int kRowsPerGroup = 128;
constexpr int kFixedCost = 4;
constexpr int kMdInts = 8;

MLA_HD inline int row_groups(int heads_per_kv) { return (heads_per_kv + kRowsPerGroup - 1) / kRowsPerGroup; }

MLA_HD inline int pages_of(int seqlen) { return seqlen <= 0 ? 0 : (seqlen + kPage - 1) / kPage; }

// seqlens: [batch]; md: [num_parts * 8]; num_splits: [batch * groups + 1].
MLA_HD inline void schedule(const int32_t* seqlens, int batch, int groups, int num_parts, int32_t* md,
                            int32_t* num_splits)
{
    const int nv = batch * groups;
    long long W = 0;
    for (int b = 0; b < batch; ++b) W += static_cast<long long>(pages_of(seqlens[b]) + kFixedCost) * groups;
    const long long T = (W + num_parts - 1) / num_parts + kFixedCost;

    num_splits[0] = 0;
    int vb = 0, blk = 0, cur_split = 0;
    for (int p = 0; p < num_parts; ++p) {
        int32_t* m = md + p * kMdInts;
        m[0] = vb;
        m[1] = blk;
        m[4] = cur_split;
        m[5] = m[6] = m[7] = 0;
        const bool last = (p == num_parts - 1);
        long long budget = T;
        while (vb < nv) {
            const int n = pages_of(seqlens[vb / groups]);
            const int rest = n - blk;
            if (rest + kFixedCost <= budget || last) {
                budget -= rest + kFixedCost;
                num_splits[vb + 1] = num_splits[vb] + cur_split + 1;
                ++vb;
                blk = 0;
                cur_split = 0;
                if (budget <= 0 && !last) break;
            } else {
                const long long take = budget - kFixedCost;
                if (take <= 0) break;
                blk += static_cast<int>(take);
                ++cur_split;
                break;
            }
        }
        m[2] = vb;
        m[3] = blk;
    }
}

}  // namespace mla
