// Tile scheduler: splits the decode work of a batch into `num_parts` contiguous
// ranges of equal cost, one per two-SM cluster of the split-KV kernel.
//
// "FlashMLA" usage page (deepep.org): get_mla_metadata analyses the sequence
// lengths once per decoding step and returns tile_scheduler_metadata and
// num_splits, reused by every layer; its Tile Scheduler "distributes work across
// GPU resources" and balances variable-length sequences ("optimized for
// variable-length sequence serving", sourcepulse summary).  The pages do not
// print the algorithm or the metadata format; this one is our own.
//
// Work units.  A "virtual batch" vb = g * batch + b is request b restricted to query
// rows [128 g, 128 g + 128) of its s_q * h_q rows.  The numbering is group-major: row
// group 0 of every request comes before row group 1 of any, so on the line below the
// groups of one request lie half a line (for two groups) apart, and the partitions that
// cover them stream the same pages at about the same time (the second read hits L2).  Every chunk (one
// partition's share of one virtual batch) costs F units of overhead (the output
// epilogue, refilling the pipeline) plus one unit per 64-token page: F = kFixedCost
// for the paged decode (kFixedCostFp8 over an FP8 cache, whose pages take about twice
// as long), kFixedCostSparse for the sparse calls, whose "pages" of 64 gathered
// entries cost two to three times a contiguous page.
// Lay the virtual batches on a line: vb takes F units followed by its pages,
// starting at C[vb] = sum of the costs before it; W is the total.  A partition
// that starts inside a virtual batch's pages opens one more chunk than the line
// shows, so it gets F units fewer of the line: with D = ceil((W - F) / num_parts),
// partition 0 takes the line units [0, F + D) and partition p >= 1 the units
// [F + p D, F + (p + 1) D); each partition's cost (pages + F per chunk) is then
// at most F + D.  D is at least F: a small batch leaves the last partitions empty rather
// than cutting its sequences into pieces smaller than a chunk's overhead.  A unit position x maps to the page position (vb, blk) with vb
// the virtual batch whose span holds x and blk = clamp(x - C[vb] - F, 0,
// pages(vb)); partition p covers the page positions from map(start p) up to
// map(start p+1).  A virtual batch whose pages are cut by partition starts is
// split; every partition computes its range on its own, so the device version
// is one thread per partition.
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
constexpr int kFixedCost = 12;       // per-chunk overhead in page units (epilogue, pipeline refill), tuned on B200
constexpr int kFixedCostFp8 = 6;     // the same for the paged decode over an FP8 cache, tuned on B200
constexpr int kFixedCostSparse = 4;  // the same for the sparse decode and prefill, tuned on B200
constexpr int kMdInts = 8;

MLA_HD inline int row_groups(int heads_per_kv) { return (heads_per_kv + kRowsPerGroup - 1) / kRowsPerGroup; }

MLA_HD inline int pages_of(int seqlen) { return seqlen <= 0 ? 0 : (seqlen + kPage - 1) / kPage; }

// Request and row group of virtual batch vb (group-major numbering, batch requests).
MLA_HD inline int vb_request(int vb, int batch) { return vb % batch; }
MLA_HD inline int vb_group(int vb, int batch) { return vb / batch; }

// Position on the page line of cost unit x.  C: exclusive prefix of the costs,
// nv entries; total: W; F: the per-chunk cost.  Returns (vb, blk) through the references.
MLA_HD inline void unit_to_page(long long x, const long long* C, const int32_t* pages, int nv, long long total,
                                int F, int& vb, int& blk)
{
    if (x >= total || nv == 0) {
        vb = nv;
        blk = 0;
        return;
    }
    if (x < 0) x = 0;
    int lo = 0, hi = nv - 1;  // largest v with C[v] <= x
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (C[mid] <= x)
            lo = mid;
        else
            hi = mid - 1;
    }
    long long b = x - C[lo] - F;
    if (b < 0) b = 0;
    vb = lo;
    blk = static_cast<int>(b);  // < pages[lo]: positions at or past the span's end belong to lo + 1
    (void)pages;
}

// Range of partition p: md row.  C / pages: per virtual batch; F: the per-chunk cost.
MLA_HD inline void partition_range(int p, int num_parts, const long long* C, const int32_t* pages, int nv,
                                   long long total, int F, int32_t* m)
{
    long long D = (total - F + num_parts - 1) / num_parts;  // line units of a partition after its first F
    // A partition shorter than one chunk's overhead would cost more than it saves: small
    // batches use fewer partitions (the rest get empty ranges) instead of one-page splits.
    if (D < F) D = F;
    auto start = [&](int q) -> long long { return q == 0 ? 0 : F + static_cast<long long>(q) * D; };
    int bv, bb, ev, eb;
    unit_to_page(start(p), C, pages, nv, total, F, bv, bb);
    if (p == num_parts - 1) {
        ev = nv;
        eb = 0;
    } else {
        unit_to_page(start(p + 1), C, pages, nv, total, F, ev, eb);
    }
    m[0] = bv;
    m[1] = bb;
    m[2] = ev;
    m[3] = eb;
    m[4] = 0;
    m[5] = m[6] = m[7] = 0;
}

// Host reference of the whole schedule (the device kernel computes the same
// values in parallel).  Scratch: C [nv] and pages [nv].
inline void schedule_host(const int32_t* seqlens, int batch, int groups, int num_parts, int F, int32_t* md,
                          int32_t* num_splits, long long* C, int32_t* pages)
{
    const int nv = batch * groups;
    long long total = 0;
    for (int v = 0; v < nv; ++v) {
        pages[v] = pages_of(seqlens[vb_request(v, batch)]);
        C[v] = total;
        total += pages[v] + F;
    }
    for (int p = 0; p < num_parts; ++p) partition_range(p, num_parts, C, pages, nv, total, F, md + p * kMdInts);
    // split counts: 1 + number of partitions that start inside a virtual batch's pages
    for (int v = 0; v <= nv; ++v) num_splits[v] = 0;
    for (int p = 0; p < num_parts; ++p) {
        int32_t* m = md + p * kMdInts;
        if (m[1] > 0) {
            // index of this split = 1 + number of earlier mid-batch starts in the same vb
            int idx = 1;
            for (int q = p - 1; q >= 0 && md[q * kMdInts + 0] == m[0] && md[q * kMdInts + 1] > 0; --q) ++idx;
            m[4] = idx;
            num_splits[m[0] + 1] += 1;  // extra splits, accumulated below
        }
    }
    int acc = 0;
    for (int v = 0; v < nv; ++v) {
        const int extra = num_splits[v + 1];
        num_splits[v] = acc;
        acc += 1 + extra;
    }
    num_splits[nv] = acc;
}

}  // namespace mla
