// MLA decoding over a paged latent KV cache on Blackwell (sm_100a).
//
// What is computed ("FlashMLA" usage page, deepep.org: flash_mla_with_kvcache;
// upstream FlashMLA documentation, "Usage / MLA Decoding" and the "MLA Mode"
// footnote): for every request b, query token s and head h,
//   o[b,s,h,:] = softmax_j(scale * q[b,s,h,:] . k_j) @ v_j,   lse = log sum_j exp(...)
// over the cached rows j the query sees, where a row is 576 (or 512) wide and
// v_j is its leading 512 columns.  The page splits the kernel into a Tile
// Scheduler, a Block Table Manager and a Memory Manager, and the work into
// Q-K product, softmax with scaling, and output; the split-KV / combine
// kernel pair is named on the "FlashMLA vLLM Optimization" page (background).
//
// Design for sm_100a (ours; the pages' kernels target Hopper):
//
// * One two-CTA cluster (an SM pair) per scheduler partition; the even CTA issues
//   two-SM tcgen05 MMAs (cta_group::2, M = 128 query rows, 64 per CTA).
//   S = Q K^T: N = 64 tokens of a page, each CTA supplying its 32 tokens (K stage of
//   32 tokens x 576 columns); O += P V: N = 256 d_v columns per MMA, each CTA supplying
//   128 of them (V stage of 64 tokens x its 256 d_v columns, read from L2 again: every
//   HBM byte is read once, every L2 byte twice).  Each CTA receives the full-width
//   results for its own 64 rows in tensor memory (the 2x2 layout of pair MMAs).
// * Tensor memory per CTA: O 256 columns, two S buffers 2 x 32, Q columns [0, 384) as
//   the A operand of Q K^T 192; shared memory: Q columns 384+, a 3-stage K ring, a
//   2-stage V ring, two P buffers (P is the A operand of P V), barriers.
// * Warp roles: 4 softmax warps (thread = TMEM lane: row t % 64, token / d_v half
//   t / 64), a K loader, the MMA issuer, a V loader (zeroes page tails), a Q loader.
//   Pages are gathered through the block table by TMA.
// * Online softmax in base 2 with a lazily moved reference maximum: O is rescaled in
//   tensor memory only when the running maximum grows by more than 2^8.
// * Epilogue: the softmax warps store the next chunk's Q into tensor memory, then drain
//   O 64 columns at a time into swizzled tiles handed to TMA bulk stores: 16-bit O for
//   unsplit chunks, fp32 partials and LSEs for split ones, which the combine kernel
//   merges as soon as each virtual batch's splits are announced.
// * The metadata, split-KV and combine kernels are launched with programmatic launch
//   overlap.
// * "FP8 with scale" cache (the kFp8 instantiation, 512 threads): the K producer bulk-copies
//   this CTA's raw 656-byte rows of each page; two converter warpgroups dequantize them
//   (e4m3 x float32 scale, rounded to bfloat16) into the K stage; the V producer assembles
//   the V stage from both CTAs' K stages with shared-memory bulk copies (its own rows
//   locally, the peer's over distributed shared memory), so every token row is dequantized
//   once and the MMA, softmax and epilogue are those of the 16-bit cache.
//
// Every mbarrier wait is bounded: after kWaitTimeoutNs the waiting thread sets
// an abort flag (seen by both CTAs of the cluster) and MLA_ERR_TIMEOUT in the
// workspace status word, and every role winds down and frees tensor memory.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/mla_decode.h"
#include "ptx.cuh"
#include "scheduler.cuh"

namespace mla {

constexpr int kThreads = 256;          // 4 softmax warps + K loader + MMA issuer + V loader + Q loader
// "FP8 with scale" cache (upstream FlashMLA documentation, "FP8 KV Cache"): 656-byte token rows
// of 512 float8_e4m3 latent values, 4 float32 scales (one per 128 latent values) and 64 bfloat16
// RoPE values.  Its kernel adds two warpgroups of converter warps that dequantize raw rows from
// shared memory into the bfloat16 K and V stages the MMAs read.
constexpr int kThreadsFp8 = 512;
constexpr int kConvWarp0 = 8;          // converter warps 8-15
constexpr int kConvWarps = 8;
constexpr int kFp8Row = 656;
constexpr int kRawKBytes = 32 * kFp8Row;       // this CTA's 32 token rows of a page, as stored
// Registers per thread in the FP8 kernel: the launch holds 65536 / 512 = 128 each; the loader /
// MMA warpgroup and the two converter warpgroups give theirs up to the softmax warpgroup.
constexpr uint32_t kRegsLaunchFp8 = 128;
constexpr uint32_t kRegsLoadersFp8 = 104;
constexpr uint32_t kRegsConvFp8 = 128;
constexpr uint32_t kRegsSoftmaxFp8 = 152;
static_assert(128 * (kRegsLoadersFp8 + kRegsSoftmaxFp8 + 2 * kRegsConvFp8) <= kThreadsFp8 * kRegsLaunchFp8,
              "register split exceeds the launch's registers");
constexpr int kKWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kVWarp = 6;
constexpr int kQWarp = 7;
constexpr int kDv = 512;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;         // O: columns [0, 256)
constexpr uint32_t kTmemS = 256;       // S buffers: [256, 288), [288, 320)
constexpr uint32_t kTmemQ = 320;       // Q columns [0, 384) as the A operand: [320, 512)
constexpr int kQTmemBoxes = 6;         // 64-column boxes of Q kept in tensor memory
constexpr int kQBoxesPerRound = 3;     // boxes of Q per round through the Q buffer
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kQPrefetchPages = 8;         // pages before a chunk's end at which the next Q goes to L2
// The bound of every pipeline wait (a build may lower it, e.g. for a test of the abort path).
#ifndef MLA_WAIT_TIMEOUT_NS
#define MLA_WAIT_TIMEOUT_NS 2000000000ull
#endif
constexpr unsigned long long kWaitTimeoutNs = MLA_WAIT_TIMEOUT_NS;
constexpr int kWorkspaceHeader = 256;
// The workspace's control block has room for the counters of this many virtual batches
// (requests x row groups of 128 query rows), whatever the call: its size does not depend on
// the problem, so the split partials of one call never overlap the counters of another.
constexpr int kMaxVirtualBatches = MLA_MAX_VIRTUAL_BATCHES;
constexpr size_t kControlBytes = kWorkspaceHeader + 2 * sizeof(int32_t) * kMaxVirtualBatches;
static_assert(kControlBytes % 256 == 0, "split partials start 256-byte aligned");
constexpr int kNumMaps = 3;  // tensor maps of the split-KV kernel: Q, K, V

// Shared-memory plan of one CTA (each CTA of the pair owns 64 query rows).  The FP8 kernel
// trades a K stage for a ring of raw cache rows.
template <bool kRope, bool kFp8 = false>
struct Layout {
    static constexpr int kBoxes = kRope ? 9 : 8;               // 64-column boxes in a d_qk row
    static constexpr int kQSmemBoxes = kBoxes - kQTmemBoxes;   // Q boxes kept in shared memory
    // the Q buffer: 64 rows, one SW128 box per 64 columns; it also stages the tensor-memory
    // part of Q, kQBoxesPerRound boxes at a time
    static constexpr int kQBytes = (kQSmemBoxes > kQBoxesPerRound ? kQSmemBoxes : kQBoxesPerRound) * 8192;
    static constexpr int kKBytes = kBoxes * 4096;              // K: this CTA's 32 tokens of a page x d_qk
    static constexpr int kKStages = kFp8 ? 2 : 3;
    static constexpr int kVBytes = 4 * 8192;                   // V: 64 tokens x this CTA's 256 d_v columns
    static constexpr int kVStages = 2;
    static constexpr int kPBytes = 8192;                       // P: 64 rows x 64 tokens, 16-bit
    static constexpr int kKSteps = kBoxes * 4;                 // K=16 MMA steps of Q K^T
    static constexpr int kRawKStages = kFp8 ? 2 : 0;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;              // kKStages stages
    static constexpr int kOffV = kOffK + kKStages * kKBytes;   // kVStages stages
    static constexpr int kOffP = kOffV + kVStages * kVBytes;   // 2 buffers
    static constexpr int kOffRawK = kOffP + 2 * kPBytes;       // raw rows (FP8 cache only)
    static constexpr int kOffRed = kOffRawK + kRawKStages * kRawKBytes;  // 3 x 128 floats: 2 page row-max halves, row sums
    static constexpr int kRedBytes = 3 * 128 * 4;
    static constexpr int kOffBar = kOffRed + kRedBytes;
    static constexpr int kBarBytes = 384;
    static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // + alignment slack
};

enum BarSlot : int {
    kBarQFull = 0,    // leader: a round of Q boxes of both CTAs landed in the Q buffer (TMA bytes)
    kBarQFree = 1,    // both: the chunk's Q K^T MMAs completed
    kBarKFull = 2,    // leader, 3 stages
    kBarKEmpty = 5,   // both, 3 stages
    kBarVFull = 8,    // leader, 2 stages: both V producers (the even one registering the TMA bytes)
    kBarVEmpty = 10,  // both, 2 stages
    kBarSFull = 12,   // both, 2 S buffers
    kBarPFull = 14,   // leader, 2 P buffers, 8 warps (4 per CTA)
    kBarPvDone = 16,  // both, 2 P buffers
    kBarOFull = 18,   // both
    kBarOFree = 19,   // leader, 8 warps
    kBarDrain = 20,   // leader
    kBarTail = 21,    // both: V load of a sequence's last page (local)
    kBarPair = 22,    // both: 2 slots, rendezvous of softmax warps {w, w ^ 2} (one arrive per warp)
    // FP8 cache only (kBarKFull then counts the converter warps of both CTAs):
    kBarRawKFull = 24,   // local, 2 stages: this CTA's raw rows of a page landed
    kBarRawKEmpty = 27,  // local, 2 stages: the converter warps done with them
    kBarKConv = 30,      // local, 2 K stages: this CTA's converter warps wrote the stage
    kBarKCopied = 32,    // local, 2 K stages: the V copies out of the stage landed (own + peer's view)
    kBarQCopied = 34,    // both: a round of Q boxes copied from the Q buffer into tensor memory
    kBarVLand = 35,      // local, 2 V stages (FP8 cache): this CTA's V stage copies landed (bytes)
    kBarCount = 37
};

// Position in a ring of kN stages: stage index and the parity of its current use.
template <int kN>
struct Ring {
    uint32_t stage = 0, phase = 0;
    __device__ void advance()
    {
        if (++stage == kN) {
            stage = 0;
            phase ^= 1u;
        }
    }
};
constexpr int kOffTmemSlot = kBarCount * 8;  // uint32 written by tcgen05.alloc
constexpr int kOffAbort = kOffTmemSlot + 4;  // int abort flag
constexpr int kOffMaskK = kOffAbort + 4;     // sparse decode: validity bits of the raw K stages' 32 rows
static_assert(kOffMaskK + 4 * Layout<true, true>::kRawKStages <= Layout<true>::kBarBytes, "barrier area too small");
static_assert(2 * Layout<true>::kPBytes >= 4 * 4096 && 2 * Layout<false>::kPBytes >= 4 * 4096,
              "epilogue staging (4 KB per softmax warp) must fit in the P buffers");
static_assert(kTmemQ + 8 * 4 * kQTmemBoxes == kTmemCols, "tensor memory plan");
static_assert(2 * kQBoxesPerRound == kQTmemBoxes && Layout<true>::kQSmemBoxes <= kQBoxesPerRound &&
                  Layout<false>::kQSmemBoxes <= kQBoxesPerRound,
              "Q goes through the Q buffer in three rounds: two into tensor memory, the rest stays");
static_assert(Layout<true>::kSmemBytes <= 232448 && Layout<false>::kSmemBytes <= 232448 &&
                  Layout<true, true>::kSmemBytes <= 232448,
              "shared memory plan exceeds 227 KB");
static_assert(Layout<true, true>::kOffK % 1024 == 0 && Layout<true, true>::kOffV % 1024 == 0 &&
                  Layout<true, true>::kOffP % 1024 == 0 && Layout<true, true>::kOffRawK % 128 == 0 &&
                  kRawKBytes % 128 == 0,
              "FP8 kernel: operand tiles 1024-byte aligned, raw rows 128-byte aligned");
static_assert(Layout<true>::kOffQ % 1024 == 0 && Layout<true>::kOffK % 1024 == 0 && Layout<true>::kOffV % 1024 == 0 &&
                  Layout<true>::kOffP % 1024 == 0 && Layout<false>::kOffK % 1024 == 0 &&
                  Layout<false>::kOffV % 1024 == 0 && Layout<false>::kOffP % 1024 == 0,
              "swizzled operand tiles must be 1024-byte aligned");

struct DecodeParams {
    const int32_t* block_table;
    const int32_t* seqlens;   // [batch]; null for the sparse decode (every request has topk entries)
    const int32_t* indices;   // sparse decode: [batch][topk] flat cache rows (page * 64 + offset), -1 invalid
    const int32_t* md;
    const int32_t* num_splits;
    const void* q;
    const void* kvcache;
    void* o;
    float* lse;
    float* max_logits;  // sparse prefill: [tokens, h_q], the largest base-2 scaled logit (null: not wanted)
    float* o_accum;     // [slots, 128, 512]
    float* lse_accum;   // [slots, 128]
    float* max_accum;   // [slots, 128] split maxima of the base-2 scaled logits
    int* status;
    int* ctl;  // [kMaxVirtualBatches][2] per virtual batch: split-KV warps that announced their
               // partials (8 per split), combine CTAs past their wait
    int batch, s_q, h_q, rows, groups, max_blocks, num_blocks, causal, box_rows;
    int active_heads;  // heads >= active_heads are padding: not written, not combined
    int o_align32;     // o is 32-byte aligned: 32-byte stores
    int topk;          // sparse decode: entries per request
    int lse_base2;     // write the LSE in base 2 (the sparse prefill's convention)
    int cache_rows;    // num_blocks * 64: a sparse entry outside [0, cache_rows) is invalid
    float scale_log2;
    int dtype, d_qk, num_parts;  // host-side dispatch only
};

// ------------------------------------------------------------------ timeline
// Built only with -DMLA_TIMELINE (the library's timeline tool builds such a copy): selected
// threads record (event id, %globaltimer ns since the CTA started) as one 32-bit word
// (id << 27 | ns) into a per-CTA, per-role slice of a device array, read back on the host
// with mla_timeline_read.  The product build compiles every TL_EV to nothing.
enum TimelineEvent : uint32_t {
    kEvSetupDone = 1,   // softmax thread 0: barriers, tensor memory and the grid dependency done
    kEvChunkBegin = 2,  // softmax thread 0: a chunk's page loop begins (its Q is in tensor memory)
    kEvSFull = 4,       // softmax thread 0: the logits of a page are ready
    kEvPPosted = 5,     // softmax thread 0: P of a page handed to the MMA
    kEvOFull = 6,       // softmax thread 0: the chunk's last P V completed
    kEvEpiDone = 7,     // softmax thread 0: the chunk's output left tensor memory
    kEvExit = 8,        // softmax thread 0: all chunks done
    kEvClusterUp = 9,   // softmax thread 0: barriers and tensor memory set up, before the grid dependency
    kEvAnnounced = 15,  // softmax thread 0: the previous split announced (epilogue start)
    kEvFirstTile = 17,  // softmax thread 0: the first 64 output columns written
    kEvTileLoaded = 19,   // softmax thread 0: 64 output columns loaded from tensor memory
    kEvMmaQFull = 10,   // MMA issuer: a chunk's Q complete
    kEvMmaKFull = 11,   // MMA issuer: a K stage landed
    kEvMmaPvGo = 12,    // MMA issuer: P and V of a page ready, P V issued
    kEvKLoad = 16,      // K producer: a K stage free, its loads issued
    kEvQLoad = 18,      // Q producer: a chunk's shared-memory Q loads issued
    kEvVLoad = 20,      // V producer: a V stage free, its loads issued
    kEvVTailLanded = 21,  // V producer: the V tile of a sequence's last page landed (before zeroing)
    kEvVTailDone = 22,    // V producer: its rows past the sequence end zeroed and the stage handed over
    kEvConvStart = 23,    // FP8 converter warp 0 (in the K producer's slice): raw rows and K stage ready
    kEvConvDone = 24,     // FP8 converter warp 0: its part of the K stage written and published
    kEvConvRaw = 25,      // FP8 converter warp 0: the page's raw rows landed
    kEvVLanded = 26,      // FP8 V producer: this CTA's V stage copies (its own and the peer's) landed
    kEvVKConv = 27,       // FP8 V producer: all converter warps of this CTA wrote the K stage
};
#ifdef MLA_TIMELINE
constexpr int kTlCtaWords = 1024;  // per CTA: 2 words of start time, then the roles' slices
constexpr int kTlMaxCtas = 160;
// Roles 0..4 (softmax, MMA, K, Q, V producers): first word and capacity of each slice.
__host__ __device__ constexpr int tl_role_base(int role)
{
    return role == 0 ? 2 : role == 1 ? 402 : role == 2 ? 802 : role == 3 ? 914 : 924;
}
__host__ __device__ constexpr int tl_role_cap(int role)
{
    return role == 0 ? 400 : role == 1 ? 400 : role == 2 ? 112 : role == 3 ? 10 : 100;
}
static_assert(tl_role_base(4) + tl_role_cap(4) == kTlCtaWords, "timeline slices fill a CTA's words");
__device__ uint32_t g_timeline[kTlMaxCtas * kTlCtaWords];
struct Timeline {
    uint32_t* buf = nullptr;
    int n = 0, cap = 0;
    uint64_t t0 = 0;
    __device__ void open(int role, uint64_t start)
    {
        t0 = start;
        if (blockIdx.x < kTlMaxCtas) {
            buf = g_timeline + blockIdx.x * kTlCtaWords + tl_role_base(role);
            cap = tl_role_cap(role);
        }
    }
    __device__ void ev(uint32_t id)
    {
        if (n < cap) buf[n++] = (id << 27) | static_cast<uint32_t>((global_timer_ns() - t0) & 0x7FFFFFFu);
    }
};
#define TL_OPEN(role) tl.open(role, tl_start)
#define TL_EV(id) tl.ev(id)
#else
struct Timeline {};
#define TL_OPEN(role) ((void)0)
#define TL_EV(id) ((void)0)
#endif

// ------------------------------------------------------------------ helpers
struct Sync {
    uint32_t abort_local;   // smem address of this CTA's abort flag
    uint32_t abort_peer;    // cluster address of the peer's abort flag
    int* status;

    __device__ bool aborted() const
    {
        int a;
        asm volatile("ld.volatile.shared.s32 %0, [%1];" : "=r"(a) : "r"(abort_local) : "memory");
        if (a) return true;
        return ld_cluster_s32(abort_peer) != 0;
    }

    __device__ void raise(int code) const
    {
        asm volatile("st.volatile.shared.s32 [%0], %1;" ::"r"(abort_local), "r"(1) : "memory");
        atomicCAS(status, 0, code);
    }

    // Bounded wait for phase `parity` of `bar`.  Returns false on abort / timeout.
    __device__ bool wait(uint32_t bar, uint32_t parity) const
    {
        if (mbar_test_wait(bar, parity)) return true;
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        const uint64_t t0 = global_timer_ns();
        while (true) {
            for (int i = 0; i < 256; ++i)
                if (mbar_try_wait(bar, parity)) return true;
            if (aborted()) return false;
            if (global_timer_ns() - t0 > kWaitTimeoutNs) {
                raise(MLA_ERR_TIMEOUT);
                return false;
            }
        }
    }
};

// Work length of request b: its cached tokens, or, for the sparse decode, its entries.
__device__ __forceinline__ int request_len(const int32_t* seqlens, int const_len, int b)
{
    return seqlens ? seqlens[b] : const_len;
}

// Iterates the chunks (vb, blk_lo, blk_hi) of one scheduler partition.
struct ChunkIter {
    int vb, blk, end_vb, end_blk, batch;
    const int32_t* seqlens;
    int const_len;  // the length of every request when seqlens is null

    __device__ bool next(int& out_vb, int& lo, int& hi)
    {
        if (!(vb < end_vb || (vb == end_vb && blk < end_blk))) return false;
        const int n = pages_of(request_len(seqlens, const_len, vb_request(vb, batch)));
        out_vb = vb;
        lo = blk;
        hi = (vb == end_vb) ? end_blk : n;
        ++vb;
        blk = 0;
        return true;
    }
};

__device__ __forceinline__ uint32_t pack2(float a, float b, bool fp16)
{
    if (fp16) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Block-table entry of page blk of a request (-1 past max_blocks).  The producers read it one
// page ahead of its use, so that its latency overlaps their wait for a free stage.
__device__ __forceinline__ int table_entry(const DecodeParams& p, const int32_t* table, int blk)
{
    return blk < p.max_blocks ? __ldg(table + blk) : -1;
}

// The cache page of a block-table entry: one outside the cache is recorded in the status word
// and replaced by page 0, so that every load stays inside the cache.
__device__ __forceinline__ int checked_page(const DecodeParams& p, int page)
{
    if (page < 0 || page >= p.num_blocks) {
        atomicCAS(p.status, 0, MLA_ERR_DEVICE_CHECK);
        page = 0;
    }
    return page;
}

// ------------------------------------------------------------------ split-KV kernel
// One cluster of two CTAs (an SM pair) per scheduler partition.  CTA c owns
// query rows [64c, 64c+64) of each 128-row group.  The even CTA issues
// two-SM tcgen05 MMAs (cta_group::2, M = 128):
//   S = Q K^T  (N = 64 tokens of a page; CTA c supplies tokens [32c, 32c+32))
//   O += P V   (N = 256 d_v columns per MMA; CTA c supplies its 128 of them)
// so each CTA receives the full logits of its own rows without any software
// exchange, and each KV byte is read from HBM once.
//
// Tensor memory of each CTA ("2x2" data-path layout of the pair MMA: lanes
// 0-63 hold the first half of N for the 64 rows, lanes 64-127 the second):
//   O   columns [0, 256):  d_v chunk i (256 wide) at [128 i, 128 i + 128)
//   S   columns [256, 288) and [288, 320): two page buffers
// Thread t of the softmax warps owns row t % 64 and token / d_v half t / 64.
template <bool kRope, bool kFp16, bool kPadHeads, bool kFp8 = false, bool kSparse = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kFp8 ? kThreadsFp8 : kThreads, 1)
    mla_splitkv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const DecodeParams p)
{
    static_assert(!kFp8 || (kRope && !kFp16), "the FP8 cache has d_qk = 576 and bfloat16 queries");
    using L = Layout<kRope, kFp8>;
    constexpr int kNumThreads = kFp8 ? kThreadsFp8 : kThreads;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_addr(smem);
    const uint32_t s_q = s_base + L::kOffQ;
    const uint32_t s_k = s_base + L::kOffK;
    const uint32_t s_v = s_base + L::kOffV;
    const uint32_t s_p = s_base + L::kOffP;
    const uint32_t s_bar = s_base + L::kOffBar;
    float* red = reinterpret_cast<float*>(smem + L::kOffRed);
    volatile uint32_t* mask_k = reinterpret_cast<volatile uint32_t*>(smem + L::kOffBar + kOffMaskK);
    [[maybe_unused]] Timeline tl;
#ifdef MLA_TIMELINE
    const uint64_t tl_start = global_timer_ns();
    if (blockIdx.x < kTlMaxCtas) {
        for (int i = 2 + threadIdx.x; i < kTlCtaWords; i += blockDim.x) g_timeline[blockIdx.x * kTlCtaWords + i] = 0;
        __syncthreads();  // the zeros land before any event of this CTA
        if (threadIdx.x == 0) {
            g_timeline[blockIdx.x * kTlCtaWords] = static_cast<uint32_t>(tl_start);
            g_timeline[blockIdx.x * kTlCtaWords + 1] = static_cast<uint32_t>(tl_start >> 32);
        }
    }
    if (threadIdx.x == 0) TL_OPEN(0);
#endif
    auto bar = [&](int slot) { return s_bar + 8u * slot; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t cta = cluster_cta_rank();
    const bool leader = (cta == 0);
    const int part = blockIdx.x >> 1;
    auto lead_bar = [&](int slot) { return map_to_cta(bar(slot), 0); };  // leader's barrier, cluster address

    // ---------------- set-up
    if (threadIdx.x == 0) {
        mbar_init(bar(kBarQFull), 1);
        mbar_init(bar(kBarQFree), 1);
        mbar_init(bar(kBarQCopied), 1);
        // K and V stages are filled by TMA (one arrival with the byte count) or, for the FP8
        // cache, by the 8 converter warps of each CTA.
        for (int s = 0; s < L::kKStages; ++s) {
            mbar_init(bar(kBarKFull + s), kFp8 ? 2 * kConvWarps : 1);
            mbar_init(bar(kBarKEmpty + s), 1);
        }
        for (int s = 0; s < L::kRawKStages; ++s) {
            mbar_init(bar(kBarRawKFull + s), 1);
            mbar_init(bar(kBarRawKEmpty + s), kConvWarps);
        }
        if constexpr (kFp8) {
            for (int s = 0; s < L::kKStages; ++s) {
                mbar_init(bar(kBarKConv + s), kConvWarps);
                mbar_init(bar(kBarKCopied + s), 2);  // this CTA's V producer and the peer's
            }
            for (int s = 0; s < L::kVStages; ++s) mbar_init(bar(kBarVLand + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(kBarVFull + s), 2);  // the V producers of both CTAs
            mbar_init(bar(kBarVEmpty + s), 1);
            mbar_init(bar(kBarSFull + s), 1);
            mbar_init(bar(kBarPFull + s), 8);
            mbar_init(bar(kBarPvDone + s), 1);
        }
        mbar_init(bar(kBarOFull), 1);
        mbar_init(bar(kBarOFree), 8);
        mbar_init(bar(kBarDrain), 1);
        mbar_init(bar(kBarTail), 1);
        mbar_init(bar(kBarPair + 0), 2);
        mbar_init(bar(kBarPair + 1), 2);
        *reinterpret_cast<volatile int*>(smem + L::kOffBar + kOffAbort) = 0;
        fence_mbar_init();
    }
    // Query rows past the loaded box stay zero (finite) for the whole kernel.
    if (p.box_rows < 64) {
        uint4* q4 = reinterpret_cast<uint4*>(smem + L::kOffQ);
        for (int i = threadIdx.x; i < L::kQBytes / 16; i += kNumThreads) q4[i] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    if (warp == kMmaWarp) {
        tmem_alloc_pair(s_bar + kOffTmemSlot, kTmemCols);
        tmem_relinquish_pair();
    }
    if (warp == kQWarp && lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers initialised before any remote arrive / transaction
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kOffBar + kOffTmemSlot);
    if (threadIdx.x == 0) TL_EV(kEvClusterUp);
    // The set-up above touched no global memory, so it may overlap the grid before this
    // one (the metadata kernel); everything below may read what that grid wrote.
    grid_dependency_wait();
    grid_launch_dependents();

    Sync sync{s_bar + kOffAbort, map_to_cta(s_bar + kOffAbort, cta ^ 1u), p.status};
    const int32_t* md = p.md + part * kMdInts;
    ChunkIter chunks{md[0], md[1], md[2], md[3], p.batch, p.seqlens, p.topk};
    const int begin_vb = md[0];
    const int begin_split = md[4];

    if (kFp8 && warp >= kConvWarp0) {
        // ============================ converters (FP8 cache) ============================
        // Eight warps per CTA dequantize this CTA's 32 raw rows of each page into the bfloat16 K
        // stage the MMAs read, in the layout TMA gives the 16-bit cache (SW128 boxes of 64
        // columns): latent value i becomes bf16(e4m3_i * scale_{i/128}) (the product in float32,
        // then rounded to nearest even), the 64 RoPE values are copied.  Rows that are not
        // visible (past the sequence end, invalid sparse entries) are written as zeros: the V
        // stages are copied from these rows, and P = 0 must never meet NaN there.  Warp cw owns
        // the 16-byte words 2 cq and 2 cq + 1 (cq = cw & 3) of K boxes [4 ch, 4 ch + 4)
        // (ch = cw >> 2) in every row `lane`.
        set_max_registers<kRegsLaunchFp8, kRegsConvFp8>();
        const int cw = warp - kConvWarp0;
        const int cq = cw & 3, ch = cw >> 2;
        const int sw = lane & 7;  // swizzle phase of row `lane` (and of every row congruent mod 8)
        const uint32_t k_full_lead = lead_bar(kBarKFull);  // + 8 per stage (slots are 8 bytes apart)
        auto wwait = [&](uint32_t b_, uint32_t par) { return __all_sync(0xffffffffu, sync.wait(b_, par)); };
        const bool tl_conv = (cw == 0 && lane == 0);
        if (tl_conv) TL_OPEN(2);
        // 16 e4m3 values (one 16-byte word) times `s` -> 16 bfloat16 values (two 16-byte words).
        // Two values at a time: e4m3 -> half (exact: every e4m3 value, subnormals and NaN
        // included, is a half), half -> float32 (exact), one packed float32 multiply by s (the
        // exact product rounded once), then the pack to bfloat16 (round to nearest even).
        auto dequant16 = [](const uint4 raw, const float s, uint4& lo, uint4& hi) {
            auto two = [s](uint32_t w16) {  // byte 0 -> low half of the result
                const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w16), __NV_E4M3);
                const float2 v = fmul2(__half22float2(*reinterpret_cast<const __half2*>(&h)), make_float2(s, s));
                const __nv_bfloat162 b = __floats2bfloat162_rn(v.x, v.y);
                return *reinterpret_cast<const uint32_t*>(&b);
            };
            auto word = [&](uint32_t w, uint32_t& a, uint32_t& b) {  // bytes 0, 1 -> a; bytes 2, 3 -> b
                a = two(w & 0xffffu);
                b = two(w >> 16);
            };
            word(raw.x, lo.x, lo.y);
            word(raw.y, lo.z, lo.w);
            word(raw.z, hi.x, hi.y);
            word(raw.w, hi.z, hi.w);
        };
        Ring<L::kKStages> kring;
        Ring<L::kRawKStages> rk;
        bool ok = true;
        int vb, lo, hi;
        while (ok && chunks.next(vb, lo, hi)) {
            if (hi <= lo) continue;
            const int Lb = request_len(p.seqlens, p.topk, vb_request(vb, p.batch));
            for (int blk = lo; blk < hi && ok; ++blk, rk.advance(), kring.advance()) {
                if (!(ok = wwait(bar(kBarRawKFull + rk.stage), rk.phase))) break;
                if (tl_conv) TL_EV(kEvConvRaw);
                // this CTA's visible rows of the page (read before the raw stage is handed back)
                uint32_t live_bits;
                if constexpr (kSparse) {
                    live_bits = mask_k[rk.stage];
                } else {
                    const int c = min(max(min(kPage, Lb - kPage * blk) - 32 * static_cast<int>(cta), 0), 32);
                    live_bits = c >= 32 ? 0xffffffffu : ((1u << c) - 1u);
                }
                // The stage is free once the Q K^T MMAs of its previous page and the V copies out
                // of it (this CTA's and the peer's) are done.
                if (!(ok = wwait(bar(kBarKEmpty + kring.stage), kring.phase ^ 1))) break;
                if (!(ok = wwait(bar(kBarKCopied + kring.stage), kring.phase ^ 1))) break;
                if (tl_conv) TL_EV(kEvConvStart);
                {
                    const bool live = (live_bits >> lane) & 1u;
                    const uint8_t* rrow = smem + L::kOffRawK + rk.stage * kRawKBytes + lane * kFp8Row;
                    uint8_t* krow = smem + L::kOffK + kring.stage * L::kKBytes + lane * 128;
                    const uint4 zero = make_uint4(0, 0, 0, 0);
                    const uint4 rope = *reinterpret_cast<const uint4*>(rrow + 528 + 16 * cw);
                    const float2 sc = *reinterpret_cast<const float2*>(rrow + 512 + 8 * ch);  // boxes 4 ch .. 4 ch + 3
                    // One box per iteration: a small loop body keeps the instruction cache warm for
                    // the other warp roles (measured faster than unrolling), and the other converter
                    // warp of the scheduler hides the load latency.
#pragma unroll 1
                    for (int m = 0; m < 4; ++m) {  // box 4 ch + m: latent columns [64 (4 ch + m), +64); 16 of them
                        uint4 w0, w1;
                        dequant16(*reinterpret_cast<const uint4*>(rrow + 64 * (4 * ch + m) + 16 * cq), m < 2 ? sc.x : sc.y,
                                  w0, w1);
                        uint8_t* box = krow + (4 * ch + m) * 4096;
                        *reinterpret_cast<uint4*>(box + (((2 * cq) ^ sw) << 4)) = w0;
                        *reinterpret_cast<uint4*>(box + (((2 * cq + 1) ^ sw) << 4)) = w1;
                    }
                    *reinterpret_cast<uint4*>(krow + 8 * 4096 + ((cw ^ sw) << 4)) = rope;  // RoPE: box 8
                    if (!live) {  // rare (a sequence's last page, invalid sparse entries): zeros over the row
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            uint8_t* box = krow + (4 * ch + m) * 4096;
                            *reinterpret_cast<uint4*>(box + (((2 * cq) ^ sw) << 4)) = zero;
                            *reinterpret_cast<uint4*>(box + (((2 * cq + 1) ^ sw) << 4)) = zero;
                        }
                        *reinterpret_cast<uint4*>(krow + 8 * 4096 + ((cw ^ sw) << 4)) = zero;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarRawKEmpty + rk.stage));
                // Visible to the tensor core and to the bulk copies (async proxy): arrive on the even
                // CTA's K_full (16 arrivals: 8 warps x 2 CTAs) and on this CTA's K_conv.
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (leader)
                        mbar_arrive(k_full_lead + 8u * kring.stage);
                    else
                        mbar_arrive_remote(k_full_lead + 8u * kring.stage);
                    mbar_arrive(bar(kBarKConv + kring.stage));
                }
                if (tl_conv) TL_EV(kEvConvDone);
            }
        }
    } else if (warp >= 4) {
        // Warpgroup 1 (Q / K / V loaders and the MMA issuer): one thread issues; few registers.
        if constexpr (kFp8) set_max_registers<kRegsLaunchFp8, kRegsLoadersFp8>();  // before the role split: one
                                                                                    // instruction per warpgroup
        if (warp == kQWarp) {
            // ============================ Q producer ============================
            // A chunk's 64 query rows go through the Q buffer (3 boxes of 64 columns) in three
            // rounds, once the previous chunk's Q K^T MMAs are done: boxes 0-2 and 3-5, which
            // the MMA warp copies into tensor memory (the A operand of columns [0, 384)), then
            // the last boxes, which stay in the buffer.  The boxes of the later rounds go to
            // L2 with the first, so their loads hit L2.
            if (lane == 0) {
                TL_OPEN(3);
                const int y_off = 64 * static_cast<int>(cta);
                uint32_t k = 0;
                int vb, lo, hi;
                bool ok = true;
                while (ok && chunks.next(vb, lo, hi)) {
                    if (hi <= lo) continue;
                    const int b = vb_request(vb, p.batch), rg = vb_group(vb, p.batch);
                    const int y = rg * kRowsPerGroup + y_off;
                    if (!(ok = sync.wait(bar(kBarQFree), (k & 1) ^ 1))) break;
                    TL_EV(kEvQLoad);
                    for (int r = 0; r < 3 && ok; ++r) {
                        const int box0 = kQBoxesPerRound * r;
                        const int nbox = r < 2 ? kQBoxesPerRound : L::kBoxes - 2 * kQBoxesPerRound;
                        if (r > 0 && !(ok = sync.wait(bar(kBarQCopied), (2 * k + r - 1) & 1))) break;
                        if (leader) mbar_arrive_expect_tx(bar(kBarQFull), 2 * nbox * p.box_rows * 128);
                        for (int i = 0; i < nbox; ++i)
                            tma_load_3d_pair(s_q + i * 8192, &tm_q, lead_bar(kBarQFull), 64 * (box0 + i), y, b);
                        if (r == 0)
                            for (int i = kQBoxesPerRound; i < L::kBoxes; ++i) tma_prefetch_3d(&tm_q, 64 * i, y, b);
                    }
                    ++k;
                }
                if (!ok) {
                    const uint64_t t0 = global_timer_ns();  // let issued loads land (see the V producer)
                    while (global_timer_ns() - t0 < 50000000ull) {
                    }
                }
            }
        } else if (warp == kKWarp) {
            // ============================ K producer ============================
            if constexpr (kSparse && kFp8) {
                static_assert(L::kRawKStages > 0, "the FP8 layout's raw ring");
                // Sparse decode: row i of this CTA's half of "page" blk is entry 64 blk + 32 cta + i
                // of the request's list.  Lane i bulk-copies its row (656 bytes as stored) when
                // the entry is valid; lane 0 records the half's validity bits with the stage and
                // registers the bytes.  Entries are read one page ahead.
                Ring<L::kRawKStages> ring;
                int vb, lo, hi;
                bool ok = true;
                const uint8_t* kv = static_cast<const uint8_t*>(p.kvcache);
                auto wwait = [&](uint32_t b_, uint32_t par) { return __all_sync(0xffffffffu, sync.wait(b_, par)); };
                while (ok && chunks.next(vb, lo, hi)) {
                    if (hi <= lo) continue;
                    const int32_t* ent = p.indices + static_cast<size_t>(vb_request(vb, p.batch)) * p.topk;
                    auto entry = [&](int blk) {
                        const int e = kPage * blk + 32 * static_cast<int>(cta) + lane;
                        return e < p.topk ? __ldg(ent + e) : -1;
                    };
                    int idx = entry(lo);
                    for (int blk = lo; blk < hi; ++blk, ring.advance()) {
                        const int idx_next = blk + 1 < hi ? entry(blk + 1) : -1;
                        const uint32_t st = ring.stage;
                        if (!(ok = wwait(bar(kBarRawKEmpty + st), ring.phase ^ 1))) break;
                        const bool valid = idx >= 0 && idx < p.cache_rows;
                        const uint32_t mask = __ballot_sync(0xffffffffu, valid);
                        if (lane == 0) {
                            mask_k[st] = mask;
                            mbar_arrive_expect_tx(bar(kBarRawKFull + st), __popc(mask) * kFp8Row);
                        }
                        __syncwarp();
                        if (valid)
                            bulk_load(s_base + L::kOffRawK + st * kRawKBytes + lane * kFp8Row,
                                      kv + static_cast<size_t>(idx) * kFp8Row, kFp8Row, bar(kBarRawKFull + st));
                        idx = idx_next;
                    }
                }
                if (!ok && lane == 0) {
                    const uint64_t t0 = global_timer_ns();  // let issued loads land (see the V producer)
                    while (global_timer_ns() - t0 < 50000000ull) {
                    }
                }
            } else if constexpr (kFp8) {
                // FP8 cache: this CTA's 32 rows of each page as stored (one bulk copy), for the
                // converters.
                if (lane == 0) {
                    Ring<L::kRawKStages> ring;
                    int vb, lo, hi;
                    bool ok = true;
                    const uint8_t* kv = static_cast<const uint8_t*>(p.kvcache);
                    while (ok && chunks.next(vb, lo, hi)) {
                        if (hi <= lo) continue;
                        const int b = vb_request(vb, p.batch);
                        const int32_t* table = p.block_table + static_cast<size_t>(b) * p.max_blocks;
                        int entry = table_entry(p, table, lo), entry_next = 0;
                        for (int blk = lo; blk < hi; ++blk, ring.advance(), entry = entry_next) {
                            entry_next = blk + 1 < hi ? table_entry(p, table, blk + 1) : 0;
                            const uint32_t st = ring.stage;
                            if (!(ok = sync.wait(bar(kBarRawKEmpty + st), ring.phase ^ 1))) break;
                            const int page = checked_page(p, entry);
                            mbar_arrive_expect_tx(bar(kBarRawKFull + st), kRawKBytes);
                            bulk_load(s_base + L::kOffRawK + st * kRawKBytes,
                                      kv + (static_cast<size_t>(page) * kPage + 32 * cta) * kFp8Row, kRawKBytes,
                                      bar(kBarRawKFull + st));
                        }
                    }
                    if (!ok) {
                        const uint64_t t0 = global_timer_ns();  // let issued loads land (see the V producer)
                        while (global_timer_ns() - t0 < 50000000ull) {
                        }
                    }
                }
            } else if constexpr (kSparse) {
                static_assert(!kFp8, "16-bit rows");
                if (lane == 0) TL_OPEN(2);
                // Sparse, 16-bit rows: row i of this CTA's half of "page" blk is entry 64 blk + 32 cta + i.
                // Lane g < 8 gathers rows 4 g .. 4 g + 3 of every 64-column box (TMA tile::gather4);
                // an invalid entry names the row just past the tensor, which reads zeros.
                Ring<L::kKStages> ring;
                int vb, lo, hi;
                bool ok = true;
                auto wwait = [&](uint32_t b_, uint32_t par) { return __all_sync(0xffffffffu, sync.wait(b_, par)); };
                while (ok && chunks.next(vb, lo, hi)) {
                    if (hi <= lo) continue;
                    const int32_t* ent = p.indices + static_cast<size_t>(vb_request(vb, p.batch)) * p.topk;
                    auto entry = [&](int blk) {
                        const int e = kPage * blk + 32 * static_cast<int>(cta) + lane;
                        const int idx = e < p.topk ? __ldg(ent + e) : -1;
                        return (idx >= 0 && idx < p.cache_rows) ? idx : p.cache_rows;
                    };
                    int row = entry(lo);
                    for (int blk = lo; blk < hi; ++blk, ring.advance()) {
                        const int row_next = blk + 1 < hi ? entry(blk + 1) : p.cache_rows;
                        const uint32_t st = ring.stage;
                        if (!(ok = wwait(bar(kBarKEmpty + st), ring.phase ^ 1))) break;
                        if (lane == 0) TL_EV(kEvKLoad);
                        if (lane == 0 && leader) mbar_arrive_expect_tx(bar(kBarKFull + st), 2 * L::kKBytes);
                        const int g = lane & 7;
                        const int r0 = __shfl_sync(0xffffffffu, row, 4 * g), r1 = __shfl_sync(0xffffffffu, row, 4 * g + 1);
                        const int r2 = __shfl_sync(0xffffffffu, row, 4 * g + 2), r3 = __shfl_sync(0xffffffffu, row, 4 * g + 3);
                        if (lane < 8)
                            for (int i = 0; i < L::kBoxes; ++i)
                                tma_gather4_pair(s_k + st * L::kKBytes + i * 4096 + 512 * g, &tm_k, lead_bar(kBarKFull + st),
                                                 64 * i, r0, r1, r2, r3);
                        row = row_next;
                    }
                }
                if (!ok && lane == 0) {
                    const uint64_t t0 = global_timer_ns();  // let issued loads land (see the V producer)
                    while (global_timer_ns() - t0 < 50000000ull) {
                    }
                }
            } else if (lane == 0) {
                TL_OPEN(2);
                Ring<L::kKStages> ring;
                int vb, lo, hi;
                bool ok = true;
#ifdef MLA_TEST_WITHHOLD_K_PAGE
                // Test-only build: both CTAs of partition 0 never load page MLA_TEST_WITHHOLD_K_PAGE
                // of their first chunk, so its K_full barrier never completes (a flag that nothing
                // sets) and the MMA warp's bounded wait on it runs out.
                bool first_chunk = true;
#endif
                while (ok && chunks.next(vb, lo, hi)) {
                    if (hi <= lo) continue;
                    const int b = vb_request(vb, p.batch);
                    const int32_t* table = p.block_table + static_cast<size_t>(b) * p.max_blocks;
#ifdef MLA_TEST_WITHHOLD_K_PAGE
                    const int withheld = (part == 0 && first_chunk) ? lo + MLA_TEST_WITHHOLD_K_PAGE : -1;
                    first_chunk = false;
#endif
                    int entry = table_entry(p, table, lo), entry_next = 0;
                    for (int blk = lo; blk < hi; ++blk, ring.advance(), entry = entry_next) {
                        entry_next = blk + 1 < hi ? table_entry(p, table, blk + 1) : 0;
                        const uint32_t st = ring.stage;
                        if (!(ok = sync.wait(bar(kBarKEmpty + st), ring.phase ^ 1))) break;
#ifdef MLA_TEST_WITHHOLD_K_PAGE
                        if (blk == withheld) continue;
#endif
                        TL_EV(kEvKLoad);
                        const int page = checked_page(p, entry);
                        if (leader) mbar_arrive_expect_tx(bar(kBarKFull + st), 2 * L::kKBytes);
                        const uint32_t dst = s_k + st * L::kKBytes;
                        for (int i = 0; i < L::kBoxes; ++i)
                            tma_load_2d_pair(dst + i * 4096, &tm_k, lead_bar(kBarKFull + st), 64 * i,
                                             page * kPage + 32 * static_cast<int>(cta));
                    }
                }
                if (!ok) {
                    const uint64_t t0 = global_timer_ns();  // let issued loads land (see the V producer)
                    while (global_timer_ns() - t0 < 50000000ull) {
                    }
                }
            }
        } else if (warp == kVWarp) {
            if constexpr (kFp8) {
                // ============================ V producer (FP8 cache) ============================
                // V(g) is the page's 64 tokens x this CTA's 256 d_v columns.  Its own 32 rows are
                // in its K stage of page g, the peer's 32 rows in the peer's (the same dequantized
                // bytes: every row is converted once).  V box jv holds K box 4 (jv >> 1) + 2 cta +
                // (jv & 1); a K box's 32 rows are 4 KB of whole SW128 rows whose swizzle phase (row
                // mod 8) is the same at token 32 c + row of the V box, so lane 0 moves each half
                // with 4 shared-memory bulk copies: into its own V stage, and into the peer's over
                // distributed shared memory, each completing on the receiving CTA's V_land.  Once
                // its V_land completes (its copies and the peer's into it), it hands the stage to
                // the MMA (the even CTA's V_full) and the K stage back to both CTAs' converters.
                if (lane == 0) {
                    TL_OPEN(4);
                    Ring<L::kKStages> kring;
                    uint32_t g = 0;
                    int vb, lo, hi;
                    bool ok = true;
                    const uint32_t peer = cta ^ 1u;
                    const uint32_t own_rows = 32u * cta * 128u;  // byte offset of this CTA's tokens in a V box
                    while (ok && chunks.next(vb, lo, hi)) {
                        if (hi <= lo) continue;
                        for (int blk = lo; blk < hi; ++blk, ++g, kring.advance()) {
                            const uint32_t vs = g & 1, vph = (g >> 1) & 1;
                            if (!(ok = sync.wait(bar(kBarKConv + kring.stage), kring.phase))) break;
                            TL_EV(kEvVKConv);
                            if (!(ok = sync.wait(bar(kBarVEmpty + vs), vph ^ 1))) break;
                            TL_EV(kEvVLoad);
                            // (the peer's stage vs is free too: the same MMA commit arrives on both CTAs)
                            mbar_arrive_expect_tx(bar(kBarVLand + vs), 2 * 4 * 4096);
                            const uint32_t kst = s_k + kring.stage * L::kKBytes;
                            const uint32_t vdst = s_v + vs * L::kVBytes + own_rows;
                            const uint32_t peer_land = map_to_cta(bar(kBarVLand + vs), peer);
                            for (int jv = 0; jv < 4; ++jv) {
                                const int mine = 4 * (jv >> 1) + 2 * static_cast<int>(cta) + (jv & 1);
                                const int theirs = 4 * (jv >> 1) + 2 * static_cast<int>(peer) + (jv & 1);
                                bulk_copy_s2c(vdst + jv * 8192, kst + mine * 4096, 4096, bar(kBarVLand + vs));
                                bulk_copy_s2c(map_to_cta(vdst + jv * 8192, peer), kst + theirs * 4096, 4096, peer_land);
                            }
                            if (!(ok = sync.wait(bar(kBarVLand + vs), vph))) break;
                            TL_EV(kEvVLanded);
                            // This CTA's copies and the peer's into it have landed: the copies out of
                            // this K stage are done, and so are the peer's out of its own.
                            mbar_arrive(bar(kBarKCopied + kring.stage));
                            mbar_arrive_remote(map_to_cta(bar(kBarKCopied + kring.stage), peer));
                            if (leader)
                                mbar_arrive(bar(kBarVFull + vs));
                            else
                                mbar_arrive_remote(lead_bar(kBarVFull + vs));
                        }
                    }
                    if (!ok) {
                        const uint64_t t0 = global_timer_ns();  // let issued copies land (see below)
                        while (global_timer_ns() - t0 < 50000000ull) {
                        }
                    }
                }
            } else if constexpr (kSparse) {
                static_assert(!kFp8, "16-bit rows");
                if (lane == 0) TL_OPEN(4);
                // ==================== V producer (sparse, 16-bit rows) ====================
                // The page's 64 entries x this CTA's 4 V boxes, by gather4 (lane g < 16: rows 4 g ..
                // 4 g + 3); invalid entries read zeros, so nothing needs clearing.
                Ring<L::kVStages> ring;
                int vb, lo, hi;
                bool ok = true;
                auto wwait = [&](uint32_t b_, uint32_t par) { return __all_sync(0xffffffffu, sync.wait(b_, par)); };
                while (ok && chunks.next(vb, lo, hi)) {
                    if (hi <= lo) continue;
                    const int32_t* ent = p.indices + static_cast<size_t>(vb_request(vb, p.batch)) * p.topk;
                    auto entry = [&](int e) {
                        const int idx = e < p.topk ? __ldg(ent + e) : -1;
                        return (idx >= 0 && idx < p.cache_rows) ? idx : p.cache_rows;
                    };
                    int row_a = entry(kPage * lo + lane), row_b = entry(kPage * lo + 32 + lane);
                    for (int blk = lo; blk < hi; ++blk, ring.advance()) {
                        const bool more = blk + 1 < hi;
                        const int next_a = more ? entry(kPage * (blk + 1) + lane) : p.cache_rows;
                        const int next_b = more ? entry(kPage * (blk + 1) + 32 + lane) : p.cache_rows;
                        const uint32_t st = ring.stage;
                        if (!(ok = wwait(bar(kBarVEmpty + st), ring.phase ^ 1))) break;
                        if (lane == 0) TL_EV(kEvVLoad);
                        if (lane == 0 && leader) mbar_arrive_expect_tx(bar(kBarVFull + st), 2 * L::kVBytes);
                        const int g = lane & 15, src = 4 * (g & 7);  // rows 4 g .. 4 g + 3 of the page
                        const int r0a = __shfl_sync(0xffffffffu, row_a, src), r1a = __shfl_sync(0xffffffffu, row_a, src + 1);
                        const int r2a = __shfl_sync(0xffffffffu, row_a, src + 2), r3a = __shfl_sync(0xffffffffu, row_a, src + 3);
                        const int r0b = __shfl_sync(0xffffffffu, row_b, src), r1b = __shfl_sync(0xffffffffu, row_b, src + 1);
                        const int r2b = __shfl_sync(0xffffffffu, row_b, src + 2), r3b = __shfl_sync(0xffffffffu, row_b, src + 3);
                        if (lane < 16) {
                            const bool hi_half = g >= 8;
                            for (int i = 0; i < 4; ++i) {
                                const int box = 4 * (i >> 1) + 2 * static_cast<int>(cta) + (i & 1);
                                tma_gather4_pair(s_v + st * L::kVBytes + i * 8192 + 512 * g, &tm_v, lead_bar(kBarVFull + st),
                                                 64 * box, hi_half ? r0b : r0a, hi_half ? r1b : r1a,
                                                 hi_half ? r2b : r2a, hi_half ? r3b : r3a);
                            }
                        }
                        __syncwarp();
                        if (lane == 0 && !leader) mbar_arrive_remote(lead_bar(kBarVFull + st));
                        row_a = next_a;
                        row_b = next_b;
                    }
                }
                if (!ok && lane == 0) {
                    const uint64_t t0 = global_timer_ns();  // let issued loads land (see below)
                    while (global_timer_ns() - t0 < 50000000ull) {
                    }
                }
            } else {
                // ============================ V producer ============================
                // Each CTA's V producer arrives once per page on the even CTA's V_full barrier.  A
                // full page: the even CTA's arrival registers both CTAs' TMA bytes, the odd one
                // arrives once its loads are issued.  A sequence's last, partial page: each CTA
                // loads its tile on a barrier of its own, zeroes the rows past the sequence end
                // (they may hold anything, NaN included, and P V must not see them) and then
                // arrives, with release semantics, as the softmax warps hand over P.  (A relaxed
                // transaction count preceded by a cluster-scope fence cost several microseconds
                // per partial page under full HBM load.)  The whole warp waits, uniformly.
                uint32_t g = 0, tails = 0;
                int vb, lo, hi;
                bool ok = true;
                if (lane == 0) TL_OPEN(4);
                auto wwait = [&](uint32_t b_, uint32_t par) { return __all_sync(0xffffffffu, sync.wait(b_, par)); };
                while (ok && chunks.next(vb, lo, hi)) {
                    if (hi <= lo) continue;
                    const int b = vb_request(vb, p.batch);
                    const int Lb = request_len(p.seqlens, p.topk, b);
                    const int tail = Lb % kPage;
                    const int last_page = pages_of(Lb) - 1;
                    const int32_t* table = p.block_table + static_cast<size_t>(b) * p.max_blocks;
                    int entry = table_entry(p, table, lo), entry_next = 0;
                    for (int blk = lo; blk < hi; ++blk, ++g, entry = entry_next) {
                        entry_next = blk + 1 < hi ? table_entry(p, table, blk + 1) : 0;
                        const uint32_t st = g & 1;
                        if (!(ok = wwait(bar(kBarVEmpty + st), ((g >> 1) & 1) ^ 1))) break;
                        if (lane == 0) TL_EV(kEvVLoad);
                        const int page = checked_page(p, entry);
                        const uint32_t dst = s_v + st * L::kVBytes;
                        const bool is_tail = (blk == last_page) && tail != 0;
                        if (!is_tail) {
                            if (lane == 0) {
                                if (leader) mbar_arrive_expect_tx(bar(kBarVFull + st), 2 * L::kVBytes);
                                for (int i = 0; i < 4; ++i) {
                                    const int box = 4 * (i >> 1) + 2 * static_cast<int>(cta) + (i & 1);
                                    tma_load_2d_pair(dst + i * 8192, &tm_v, lead_bar(kBarVFull + st), 64 * box, page * kPage);
                                }
                                if (!leader) mbar_arrive_remote(lead_bar(kBarVFull + st));
                            }
                        } else {
                            if (lane == 0) {
                                mbar_arrive_expect_tx(bar(kBarTail), L::kVBytes);
                                for (int i = 0; i < 4; ++i) {
                                    const int box = 4 * (i >> 1) + 2 * static_cast<int>(cta) + (i & 1);
                                    tma_load_2d(dst + i * 8192, &tm_v, bar(kBarTail), 64 * box, page * kPage);
                                }
                            }
                            if (!(ok = wwait(bar(kBarTail), tails & 1))) break;
                            if (lane == 0) TL_EV(kEvVTailLanded);
                            ++tails;
                            // rows [tail, 64) of each of the 4 boxes: contiguous bytes [tail*128, 8192)
                            for (int box = 0; box < 4; ++box) {
                                uint4* z = reinterpret_cast<uint4*>(smem + L::kOffV + st * L::kVBytes + box * 8192 +
                                                                    tail * 128);
                                for (int w16 = lane; w16 < (kPage - tail) * 8; w16 += 32) z[w16] = make_uint4(0, 0, 0, 0);
                            }
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                if (leader)
                                    mbar_arrive(bar(kBarVFull + st));
                                else
                                    mbar_arrive_remote(lead_bar(kBarVFull + st));
                                TL_EV(kEvVTailDone);
                            }
                        }
                    }
                }
                if (!ok && lane == 0) {
                    // Give loads already issued (they complete on the even CTA's barriers) time
                    // to land before shared memory goes away.
                    const uint64_t t0 = global_timer_ns();
                    while (global_timer_ns() - t0 < 50000000ull) {
                    }
                }
            }
        } else if (warp == kMmaWarp) {
            // ============================ MMA issuer (even CTA) ============================
            // The whole warp runs the loop (so addresses and descriptors stay warp-uniform);
            // one elected lane issues each tcgen05 instruction.
            if (leader) {
                constexpr uint32_t idesc_qk = instr_desc_f16(kFp16, 128, 64, false);
                constexpr uint32_t idesc_pv = instr_desc_f16(kFp16, 128, 256, true);
                constexpr uint16_t both = 0x3;
                // Base descriptors; a K step or a stage moves the start address, which is
                // the low field of the descriptor (address >> 4).
                const uint64_t q_desc = smem_desc(s_q, 16, 1024, kLayoutSW128);
                const uint64_t k_desc = smem_desc(s_k, 16, 1024, kLayoutSW128);
                const uint64_t p_desc = smem_desc(s_p, 16, 1024, kLayoutSW128);
                const uint64_t v_desc = smem_desc(s_v, 8192, 1024, kLayoutSW128);
                const bool issuer = elect_one();
                if (issuer) TL_OPEN(1);
                auto wwait = [&](uint32_t b_, uint32_t par) { return __all_sync(0xffffffffu, sync.wait(b_, par)); };
                uint32_t g = 0, k = 0;
                int vb, lo, hi;
                bool ok = true;
                auto issue_pv = [&](uint32_t gp, bool first) -> bool {
                    const uint32_t pb = gp & 1;
                    if (!wwait(bar(kBarPFull + pb), (gp >> 1) & 1)) return false;
                    if (first && !wwait(bar(kBarOFree), (k & 1) ^ 1)) return false;
                    // V stage of page gp (one stage for the FP8 cache, else it pairs with the P buffer)
                    const uint32_t vs = L::kVStages == 1 ? 0u : pb;
                    const uint32_t vpar = L::kVStages == 1 ? (gp & 1) : ((gp >> 1) & 1);
                    if (!wwait(bar(kBarVFull + vs), vpar)) return false;
                    tc_fence_after();
                    if (issuer) {
                        TL_EV(kEvMmaPvGo);
                        const uint64_t pd0 = p_desc + ((pb * L::kPBytes) >> 4);
                        const uint64_t vd0 = v_desc + ((vs * L::kVBytes) >> 4);
    #pragma unroll
                        for (int i = 0; i < 2; ++i) {
    #pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                // A = P[64 rows, 16 tokens] K-major; B = V[16 tokens, 128 d_v] of this CTA,
                                // MN-major: 64-column boxes 8 KB apart (LBO), 8-token groups 1 KB apart (SBO).
                                mma_ss_pair(tmem + kTmemO + 128 * i, pd0 + ((kk * 32) >> 4),
                                            vd0 + ((2 * i * 8192 + kk * 2048) >> 4), idesc_pv,
                                            (first && kk == 0) ? 0u : 1u);
                            }
                        }
                        mma_commit_pair(bar(kBarVEmpty + vs), both);
                        mma_commit_pair(bar(kBarPvDone + pb), both);
                    }
                    __syncwarp();
                    return true;
                };
                Ring<L::kKStages> kring;
                while (ok && chunks.next(vb, lo, hi)) {
                    const int n = hi - lo;
                    if (n <= 0) continue;
                    // rounds 0 and 1 of the chunk's Q: from the Q buffer into tensor memory (a
                    // 16-byte column slice per copy), ordered before the MMAs that read them
                    for (int r = 0; r < 2 && ok; ++r) {
                        if (!(ok = wwait(bar(kBarQFull), (3 * k + r) & 1))) break;
                        tc_fence_after();
                        if (issuer) {
#pragma unroll
                            for (int i = 0; i < kQBoxesPerRound; ++i)
#pragma unroll
                                for (int j = 0; j < 8; ++j)
                                    tmem_cp_64x128_pair(tmem + kTmemQ + 32 * (kQBoxesPerRound * r + i) + 4 * j,
                                                        q_desc + ((i * 8192 + 16 * j) >> 4));
                            mma_commit_pair(bar(kBarQCopied), both);
                        }
                        __syncwarp();
                    }
                    if (!ok || !(ok = wwait(bar(kBarQFull), (3 * k + 2) & 1))) break;
                    if (issuer) TL_EV(kEvMmaQFull);
                    for (int j = 0; j < n && ok; ++j, kring.advance()) {
                        const uint32_t gp = g + j;
                        const uint32_t sb = gp & 1;
                        const uint32_t st = kring.stage;
                        if (!(ok = wwait(bar(kBarKFull + st), kring.phase))) break;
                        tc_fence_after();
                        if (issuer) {
                            TL_EV(kEvMmaKFull);
                            const uint64_t kd0 = k_desc + ((st * L::kKBytes) >> 4);
                            // Q columns [0, 384) from tensor memory (8 columns per K=16 step) ...
    #pragma unroll
                            for (int ks = 0; ks < 4 * kQTmemBoxes; ++ks)
                                mma_ts_pair(tmem + kTmemS + 32 * sb, tmem + kTmemQ + 8 * ks,
                                            kd0 + (((ks >> 2) * 4096 + (ks & 3) * 32) >> 4), idesc_qk, ks > 0 ? 1u : 0u);
                            // ... and the remaining columns from shared memory.
    #pragma unroll
                            for (int ks = 4 * kQTmemBoxes; ks < L::kKSteps; ++ks) {
                                const int box = ks >> 2, sub = ks & 3;
                                mma_ss_pair(tmem + kTmemS + 32 * sb, q_desc + (((box - kQTmemBoxes) * 8192 + sub * 32) >> 4),
                                            kd0 + ((box * 4096 + sub * 32) >> 4), idesc_qk, 1u);
                            }
                            mma_commit_pair(bar(kBarKEmpty + st), both);
                            mma_commit_pair(bar(kBarSFull + sb), both);
                            if (j == n - 1) mma_commit_pair(bar(kBarQFree), both);
                        }
                        __syncwarp();
                        if (j > 0) ok = issue_pv(gp - 1, j == 1);
                    }
                    if (ok) ok = issue_pv(g + n - 1, n == 1);
                    if (ok && issuer) mma_commit_pair(bar(kBarOFull), both);
                    __syncwarp();
                    g += n;
                    ++k;
                }
                // Every issued MMA completes before tensor memory is released.
                if (issuer) {
                    mma_commit_pair(bar(kBarDrain), 0x1);
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar(kBarDrain), 0) && global_timer_ns() - t0 < 100000000ull) {
                    }
                }
                __syncwarp();
            }
        }
    } else {
        if constexpr (kFp8) set_max_registers<kRegsLaunchFp8, kRegsSoftmaxFp8>();
        // ======================= softmax / correction / epilogue =======================
        const int t = threadIdx.x;             // TMEM lane
        const int r = t & 63;                  // row within this CTA's 64
        const int h = t >> 6;                  // token half of S, d_v half of each O chunk
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t pair_bar = bar(kBarPair + (warp & 1));  // rendezvous of warps {w, w ^ 2}
        uint32_t pair_phase = 0;
        const uint32_t p_full_lead = lead_bar(kBarPFull);  // + 8 per P buffer
        const uint32_t o_free_lead = lead_bar(kBarOFree);
        auto wwait = [&](uint32_t b_, uint32_t par) { return __all_sync(0xffffffffu, sync.wait(b_, par)); };
        auto q_row_ptr = [&](int qvb, bool& valid) {
            const int qrow_idx = vb_group(qvb, p.batch) * kRowsPerGroup + 64 * static_cast<int>(cta) + r;
            valid = qrow_idx < p.rows;
            return reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.q) +
                                                  (static_cast<size_t>(vb_request(qvb, p.batch)) * p.rows + qrow_idx) * p.d_qk * 2);
        };
        // The whole row (the tensor-memory columns this warp stores and the shared-memory
        // ones the Q producer loads), once per row: threads t and t ^ 64 share it.
        auto prefetch_q_row = [&](int qvb) {
            bool valid;
            const uint8_t* a = reinterpret_cast<const uint8_t*>(q_row_ptr(qvb, valid));
            if (valid && h == 0)
                for (int i = 0; i < p.d_qk * 2 / 128; ++i) prefetch_l2(a + 128 * i);
        };
        uint32_t g = 0, k = 0;
        int vb, lo, hi;
        bool ok = true;
        // The combine of a virtual batch starts once the 8 warps of each of its splits (4 per
        // CTA of the pair) have announced their partial results.  A warp announces a split
        // at the start of its next epilogue, or at the end, when its stores have long
        // completed, so the fences before the announcement cost little.
        int announce_vb = -1;
        auto announce = [&]() {
            if (announce_vb >= 0) {
                __threadfence();  // this lane's partial-output and LSE stores of that split ...
                __syncwarp();
                if (lane == 0) {
                    __threadfence();  // ... and the whole warp's, before the counter update
                    atomicAdd(p.ctl + 2 * announce_vb, 1);
                }
                __syncwarp();
                announce_vb = -1;
            }
        };
        if (t == 0) TL_EV(kEvSetupDone);
        bool have = chunks.next(vb, lo, hi);
        while (ok && have) {
            const int b = vb_request(vb, p.batch), rg = vb_group(vb, p.batch);
            const int Lb = request_len(p.seqlens, p.topk, b);
            const int row = rg * kRowsPerGroup + 64 * static_cast<int>(cta) + r;
            const bool row_valid = row < p.rows;
            const int s_tok = row / p.h_q;
            int n_vis = Lb;
            if (p.causal) n_vis = min(max(Lb - p.s_q + 1 + s_tok, 0), Lb);
            const int nsplit = p.num_splits[vb + 1] - p.num_splits[vb];
            const int split_idx = (vb == begin_vb) ? begin_split : 0;
            const size_t slot = static_cast<size_t>(p.num_splits[vb]) + split_idx;  // split partial's workspace slot
            const int n = hi - lo;
            float m_ref = -INFINITY, l_half = 0.f;
            float row_max = -INFINITY;  // the chunk's largest scaled logit, base 2 (the prefill's max_logits)

            if (t == 0) TL_EV(kEvChunkBegin);
            // The next chunk's Q row goes to L2 a few pages before the end of this chunk, so
            // that loading it at the transition hits L2 (earlier, the KV stream through L2
            // would evict it again).
            const int j_prefetch = max(0, n - kQPrefetchPages);
            // Sparse decode: a page's visible columns are its valid entries.  Lane i of this warp
            // reads entry 64 page + 32 h + i (one page ahead) and a ballot gives the warp's 32 bits.
            const int32_t* ent = kSparse ? p.indices + static_cast<size_t>(b) * p.topk : nullptr;
            auto entry = [&](int blk) {
                const int e = kPage * blk + 32 * h + lane;
                return e < p.topk ? __ldg(ent + e) : -1;
            };
            int sp_idx = (kSparse && n > 0) ? entry(lo) : -1;

            for (int j = 0; j < n; ++j) {
                if (j == j_prefetch) {
                    ChunkIter peek = chunks;
                    int pvb, plo, phi;
                    while (peek.next(pvb, plo, phi))
                        if (phi > plo) {
                            prefetch_q_row(pvb);
                            break;
                        }
                }
                const uint32_t gp = g + j;
                const uint32_t sb = gp & 1;
                if (!(ok = wwait(bar(kBarSFull + sb), (gp >> 1) & 1))) break;
                if (t == 0) TL_EV(kEvSFull);
                tc_fence_after();
                // Logits stay unscaled until the exponent: scale > 0 keeps the maximum, and
                // scale * s - ref is one FFMA.  Only a page the row does not fully see
                // (the sequence's last page, the causal diagonal) needs the mask.
                float x[32];
                {
                    uint32_t vis = 0xffffffffu;  // visible columns (bit c: column 32 h + c)
                    if constexpr (kSparse) {
                        const int sp_next = (j + 1 < n) ? entry(lo + j + 1) : -1;
                        vis = __ballot_sync(0xffffffffu, sp_idx >= 0 && sp_idx < p.cache_rows);
                        sp_idx = sp_next;
                    }
                    uint32_t a[32];
                    tmem_ld32(tmem + kTmemS + 32 * sb + lane_base, a);
                    tmem_wait_ld();
                    reg_fence(a);
                    if constexpr (!kSparse) {
                        const int lim = n_vis - (lo + j) * kPage - 32 * h;  // columns >= lim are not visible
                        vis = lim >= 32 ? 0xffffffffu : (lim <= 0 ? 0u : ((1u << lim) - 1u));
                    }
                    if (__all_sync(0xffffffffu, vis == 0xffffffffu)) {
#pragma unroll
                        for (int c = 0; c < 32; ++c) x[c] = __uint_as_float(a[c]);
                    } else {
#pragma unroll
                        for (int c = 0; c < 32; ++c) x[c] = ((vis >> c) & 1u) ? __uint_as_float(a[c]) : -INFINITY;
                    }
                }
                float mx;
                {
                    float m16[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c) m16[c] = fmaxf(x[c], x[c + 16]);
#pragma unroll
                    for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
                        for (int c = 0; c < w; ++c) m16[c] = fmaxf(m16[c], m16[c + w]);
                    mx = m16[0] * p.scale_log2;  // log2-domain maximum (-inf stays -inf)
                }
                red[sb * 128 + t] = mx;
                __syncwarp();
                if (lane == 0) mbar_arrive(pair_bar);
                if (!(ok = wwait(pair_bar, pair_phase++ & 1))) break;
                mx = fmaxf(mx, red[sb * 128 + (t ^ 64)]);
                row_max = fmaxf(row_max, mx);
                // the same decision in both halves of the row
                float alpha = 1.f;
                bool rescale = false;
                if (mx > m_ref + kRescaleThreshold) {
                    if (m_ref != -INFINITY) {
                        alpha = fast_exp2(m_ref - mx);
                        rescale = (j > 0);
                    }
                    m_ref = mx;
                }
                const float ref = (m_ref == -INFINITY) ? 0.f : m_ref;
                uint32_t pk[16];
                float s16[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float p0 = fast_exp2(fmaf(x[2 * c], p.scale_log2, -ref));
                    const float p1 = fast_exp2(fmaf(x[2 * c + 1], p.scale_log2, -ref));
                    s16[c] = p0 + p1;
                    pk[c] = pack2(p0, p1, kFp16);
                }
#pragma unroll
                for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
                    for (int c = 0; c < w; ++c) s16[c] += s16[c + w];
                const float rs = s16[0];
                l_half = l_half * alpha + rs;

                if (__any_sync(0xffffffffu, rescale)) {
                    // every earlier PV has completed before O is touched
                    if (!(ok = wwait(bar(kBarPvDone + ((gp - 1) & 1)), ((gp - 1) >> 1) & 1))) break;
                    tc_fence_after();
                    const float a = rescale ? alpha : 1.f;
#pragma unroll 1
                    for (int cb = 0; cb < 8; ++cb) {
                        uint32_t v[32];
                        const uint32_t addr = tmem + kTmemO + lane_base + 32 * cb;
                        tmem_ld32(addr, v);
                        tmem_wait_ld();
                        reg_fence(v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * a);
                        tmem_st32(addr, v);
                    }
                    tmem_wait_st();
                }
                // P buffer gp&1 was last read by the PV of page gp-2.  That PV was issued
                // before the Q K^T of page gp, tcgen05 MMAs of one thread complete in
                // issue order, and the S_full commit of page gp covers every earlier MMA:
                // having waited for S_full, the buffer is free.
                {
                    uint8_t* prow = smem + L::kOffP + sb * L::kPBytes + r * 128;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int chunk = (4 * h + q) ^ (r & 7);
                        *reinterpret_cast<uint4*>(prow + chunk * 16) =
                            make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (leader)
                        mbar_arrive(bar(kBarPFull + sb));
                    else
                        mbar_arrive_remote(p_full_lead + 8u * sb);
                }
                if (t == 0) TL_EV(kEvPPosted);
            }
            if (!ok) break;

            // (The next chunk's Q reaches tensor memory without these warps: the Q producer
            // and the MMA warp move it while this epilogue drains O.)
            int nvb = 0, nlo = 0, nhi = 0;
            const bool have_next = chunks.next(nvb, nlo, nhi);

            // ---- epilogue: full row sum from both halves, O / l, LSE
            const bool empty = (n <= 0);
            red[256 + t] = l_half;
            __syncwarp();
            if (lane == 0) mbar_arrive(pair_bar);
            if (!(ok = wwait(pair_bar, pair_phase++ & 1))) break;
            const float l_other = red[256 + (t ^ 64)];
            const float l_sum = (h == 0) ? (l_half + l_other) : (l_other + l_half);
            __syncwarp();
            if (lane == 0) mbar_arrive(pair_bar);  // red[256..] free for the next chunk once both have read it
            if (!(ok = wwait(pair_bar, pair_phase++ & 1))) break;
            const float inv_l = (l_sum > 0.f) ? 1.f / l_sum : 0.f;
            const float lse2 = (l_sum > 0.f) ? m_ref + log2f(l_sum) : -INFINITY;  // base 2
            const float lse_v = lse2 * 0.69314718055994531f;                        // natural log
            if (!empty) {
                if (!(ok = wwait(bar(kBarOFull), k & 1))) break;
                if (t == 0) TL_EV(kEvOFull);
                tc_fence_after();
            }
            announce();
            if (t == 0) TL_EV(kEvAnnounced);
            // O leaves tensor memory 64 columns at a time and goes straight from registers to
            // global memory: each lane writes its row's 64 values with 32-byte stores (whole
            // sectors).  No staging tile, no TMA unit (whose queue is shared with the
            // producers' loads), nothing to wait for.  Rows past the end and padding heads are
            // skipped.
            {
                const int row_g = 64 * static_cast<int>(cta) + (t & 32) + lane;  // this lane's row in the group
                const int grow = rg * kRowsPerGroup + row_g;
                const bool live = grow < p.rows && (!kPadHeads || grow % p.h_q < p.active_heads);
                uint8_t* const o_row = static_cast<uint8_t*>(p.o) + (static_cast<size_t>(b) * p.rows + grow) * (kDv * 2);
                float* const acc_row = p.o_accum + (slot * kRowsPerGroup + row_g) * static_cast<size_t>(kDv);
#pragma unroll 1
                for (int blk2 = 0; blk2 < 4; ++blk2) {
                    // two 32-column TMEM loads in flight per wait
                    uint32_t v2[2][32];
                    if (!empty) {
                        tmem_ld32(tmem + kTmemO + 64 * blk2 + lane_base, v2[0]);
                        tmem_ld32(tmem + kTmemO + 64 * blk2 + 32 + lane_base, v2[1]);
                        tmem_wait_ld();
                        reg_fence(v2[0]);
                        reg_fence(v2[1]);
                        if (t == 0) TL_EV(kEvTileLoaded);
                        if (blk2 == 3) {
                            // O has left tensor memory: the next chunk's P V may start
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) {
                                if (leader)
                                    mbar_arrive(bar(kBarOFree));
                                else
                                    mbar_arrive_remote(o_free_lead);
                            }
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) v2[0][e] = v2[1][e] = 0;
                    }
                    const int col0 = 256 * (blk2 >> 1) + 128 * h + 64 * (blk2 & 1);  // first d_v column
                    if (live) {
                        if (nsplit == 1) {
#pragma unroll
                            for (int c = 0; c < 4; ++c) {  // 16 values (32 bytes) per store
                                const uint32_t* v = v2[c >> 1] + 16 * (c & 1);
                                uint32_t w[8];
#pragma unroll
                                for (int i = 0; i < 8; ++i)
                                    w[i] = pack2(__uint_as_float(v[2 * i]) * inv_l, __uint_as_float(v[2 * i + 1]) * inv_l, kFp16);
                                st_global_32B(o_row + (col0 + 16 * c) * 2, w, p.o_align32);
                            }
                        } else {
#pragma unroll
                            for (int c = 0; c < 8; ++c) {  // 8 values (32 bytes) per store
                                const uint32_t* v = v2[c >> 2] + 8 * (c & 3);
                                uint32_t w[8];
#pragma unroll
                                for (int i = 0; i < 8; ++i) w[i] = __float_as_uint(__uint_as_float(v[i]) * inv_l);
                                st_global_32B(acc_row + col0 + 8 * c, w, true);
                            }
                        }
                    }
                    if (blk2 == 0 && t == 0) TL_EV(kEvFirstTile);
                }
            }
            if (t == 0) TL_EV(kEvEpiDone);
            if (h == 0 && row_valid && (!kPadHeads || row % p.h_q < p.active_heads)) {
                if (nsplit == 1) {
                    const size_t at = static_cast<size_t>(b) * p.rows + row;
                    p.lse[at] = p.lse_base2 ? lse2 : lse_v;
                    if (p.max_logits) p.max_logits[at] = row_max;
                } else {
                    p.lse_accum[slot * kRowsPerGroup + 64 * cta + r] = lse_v;
                    p.max_accum[slot * kRowsPerGroup + 64 * cta + r] = row_max;
                }
            }
            if (nsplit > 1) announce_vb = vb;
            if (!empty) ++k;
            g += (n > 0 ? n : 0);
            have = have_next;
            vb = nvb;
            lo = nlo;
            hi = nhi;
        }
        if (ok) announce();
        if (t == 0) TL_EV(kEvExit);
    }

    // ---------------- teardown
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no remote access to this CTA and no MMA in flight after this point
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ combine kernel
// Merges the split partial results of every virtual batch with more than one
// split: lse = log sum_k exp(lse_k), o = sum_k exp(lse_k - lse) o_k (the exact
// identity behind split-KV).  Two layouts of the same sum, chosen on the host:
//  * few splits per virtual batch: one warp per query row, 4 rows per CTA; lane i
//    owns 16 of the 512 output columns and walks the splits in order;
//  * many splits (few virtual batches, long sequences): one CTA per row, warp w
//    sums splits w, w + 4, ... and the four partial sums are added through shared
//    memory, so a row's splits are read four at a time.
template <bool kFp16, bool kSplitParallel>
__global__ void __launch_bounds__(128) mla_combine_kernel(DecodeParams p)
{
    // No wait for the whole split-KV grid: the CTAs of a virtual batch start combining once
    // its splits are announced (8 warps per split), while other partitions still run.  This
    // grid is launched only after every split-KV CTA is resident (programmatic launch), so
    // the wait below cannot starve its producers; it is bounded all the same.  The last
    // combine CTA of the virtual batch past the wait clears both counters for the next call.
    // (The schedule was written by the metadata grid, complete before the split-KV grid
    // allowed this one to launch.)
    const int vb = blockIdx.x;
    const int slot0 = p.num_splits[vb];
    const int nsplit = p.num_splits[vb + 1] - slot0;
    if (nsplit <= 1) return;
    __shared__ int go;
    if (threadIdx.x == 0) {
        const int want = 8 * nsplit;
        int* split_done = p.ctl + 2 * vb;
        int* combine_passed = split_done + 1;
        bool ready = ld_acquire_gpu(split_done) >= want;
        const uint64_t t0 = global_timer_ns();
        while (!ready) {
            __nanosleep(200);
            ready = ld_acquire_gpu(split_done) >= want;
            // A device error recorded by this call (a split-KV cluster that gave up, another
            // combine CTA that timed out) means the splits may never all come: stop waiting.
            if (!ready && ld_acquire_gpu(p.status) != 0) break;
            if (!ready && global_timer_ns() - t0 > kWaitTimeoutNs) {
                atomicCAS(p.status, 0, MLA_ERR_TIMEOUT);
                break;
            }
        }
        if (ready && atomicAdd(combine_passed, 1) == static_cast<int>(gridDim.y) - 1) {
            *combine_passed = 0;
            *split_done = 0;
        }
        go = ready;
    }
    __syncthreads();
    if (!go) return;
    const int b = vb_request(vb, p.batch), rg = vb_group(vb, p.batch);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = kSplitParallel ? static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.y) * 4 + warp;
    const int rows_here = min(kRowsPerGroup, p.rows - rg * kRowsPerGroup);
    // uniform over the CTA in the split-parallel layout; padding heads are not combined
    if (r >= rows_here || (rg * kRowsPerGroup + r) % p.h_q >= p.active_heads) return;
    const float* lse_k = p.lse_accum + static_cast<size_t>(slot0) * kRowsPerGroup + r;
    const float* max_k = p.max_accum + static_cast<size_t>(slot0) * kRowsPerGroup + r;
    // The splits' LSEs (and maxima) are read once, in one round trip: lane i holds splits i,
    // i + 32 and i + 64 (a virtual batch has at most one split per partition; further splits,
    // for a caller's partition count above 96, are read again where needed).
    constexpr int kLseRegs = 3;
    float lk[kLseRegs], mk[kLseRegs];
#pragma unroll
    for (int i = 0; i < kLseRegs; ++i) {
        const int k = lane + 32 * i;
        lk[i] = k < nsplit ? __ldcg(lse_k + static_cast<size_t>(k) * kRowsPerGroup) : -INFINITY;
        mk[i] = (p.max_logits && k < nsplit) ? __ldcg(max_k + static_cast<size_t>(k) * kRowsPerGroup) : -INFINITY;
    }
    float mx = fmaxf(fmaxf(lk[0], lk[1]), lk[2]);
    float row_max = fmaxf(fmaxf(mk[0], mk[1]), mk[2]);  // the largest base-2 scaled logit (the prefill's max_logits)
    for (int k = lane + 32 * kLseRegs; k < nsplit; k += 32) {
        mx = fmaxf(mx, __ldcg(lse_k + static_cast<size_t>(k) * kRowsPerGroup));
        if (p.max_logits) row_max = fmaxf(row_max, __ldcg(max_k + static_cast<size_t>(k) * kRowsPerGroup));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        row_max = fmaxf(row_max, __shfl_xor_sync(0xffffffffu, row_max, o));
    }
    float sum = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
        for (int i = 0; i < kLseRegs; ++i) sum += expf(lk[i] - mx);  // exp(-inf) = 0 for absent splits
        for (int k = lane + 32 * kLseRegs; k < nsplit; k += 32) sum += expf(__ldcg(lse_k + static_cast<size_t>(k) * kRowsPerGroup) - mx);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float lse = (mx == -INFINITY) ? -INFINITY : mx + logf(sum);
    // weight of split k = exp(lse_k - lse), from lane k % 32's registers (k warp-uniform)
    float wk[kLseRegs];
#pragma unroll
    for (int i = 0; i < kLseRegs; ++i) wk[i] = expf(lk[i] - lse);
    auto weight = [&](int k) {
        if (k >= 32 * kLseRegs) return expf(__ldcg(lse_k + static_cast<size_t>(k) * kRowsPerGroup) - lse);
        const float w = k < 32 ? wk[0] : (k < 64 ? wk[1] : wk[2]);
        return __shfl_sync(0xffffffffu, w, k & 31);
    };
    float4 acc[4];  // float4 columns lane, lane + 32, lane + 64, lane + 96
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    auto fma4 = [](float4& a, const float4& v, float w) {
        a.x += w * v.x; a.y += w * v.y; a.z += w * v.z; a.w += w * v.w;
    };
    if (mx != -INFINITY) {
        const float4* src = reinterpret_cast<const float4*>(p.o_accum + (static_cast<size_t>(slot0) * kRowsPerGroup + r) * kDv) + lane;
        const size_t stride4 = static_cast<size_t>(kRowsPerGroup) * kDv / 4;  // float4s between splits
        // Splits k0, k0 + step, ... (up to 4 at a time): all their partials in flight at once.
        auto add_splits = [&](int k0, int step) {
            float4 v[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int k = k0 + step * j;
                if (k < nsplit) {
                    const float4* s4 = src + static_cast<size_t>(k) * stride4;
                    v[j][0] = __ldcg(s4);
                    v[j][1] = __ldcg(s4 + 32);
                    v[j][2] = __ldcg(s4 + 64);
                    v[j][3] = __ldcg(s4 + 96);
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int k = k0 + step * j;
                if (k < nsplit) {
                    const float w = weight(k);
#pragma unroll
                    for (int i = 0; i < 4; ++i) fma4(acc[i], v[j][i], w);
                }
            }
        };
        if (kSplitParallel) {
#pragma unroll 1
            for (int kb = warp; kb < nsplit; kb += 16) add_splits(kb, 4);  // this warp's splits warp, warp + 4, ...
        } else {
#pragma unroll 1
            for (int kb = 0; kb < nsplit; kb += 4) add_splits(kb, 1);
        }
    }
    if (kSplitParallel) {
        __shared__ float4 part[3][128];  // warps 1-3's sums
        if (warp > 0)
#pragma unroll
            for (int i = 0; i < 4; ++i) part[warp - 1][lane + 32 * i] = acc[i];
        __syncthreads();
        if (warp != 0) return;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int w = 0; w < 3; ++w) {
                const float4 o = part[w][lane + 32 * i];
                acc[i].x += o.x; acc[i].y += o.y; acc[i].z += o.z; acc[i].w += o.w;
            }
    }
    const int row = rg * kRowsPerGroup + r;
    uint2* dst = reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.o) + (static_cast<size_t>(b) * p.rows + row) * kDv * 2);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        dst[lane + 32 * i] = make_uint2(pack2(acc[i].x, acc[i].y, kFp16), pack2(acc[i].z, acc[i].w, kFp16));
    if (lane == 0) {
        const size_t at = static_cast<size_t>(b) * p.rows + row;
        p.lse[at] = p.lse_base2 ? lse * 1.4426950408889634f : lse;
        if (p.max_logits) p.max_logits[at] = row_max;
    }
}

// ------------------------------------------------------------------ metadata kernel
// Exclusive prefix sum over n values held in shared memory, by one CTA.
template <typename T>
__device__ void block_exclusive_scan(T* data, int n, T* warp_tot, T& total)
{
    const int tid = threadIdx.x, nt = blockDim.x;
    const int per = (n + nt - 1) / nt;
    const int lo = min(n, tid * per), hi = min(n, lo + per);
    T local = 0;
    for (int i = lo; i < hi; ++i) local += data[i];
    // inclusive scan of the per-thread sums across the block
    T x = local;
    const int lane = tid & 31, w = tid >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const T y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[w] = x;
    __syncthreads();
    if (w == 0) {
        T t = (lane < (nt >> 5)) ? warp_tot[lane] : T(0);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const T y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        if (lane < (nt >> 5)) warp_tot[lane] = t;
    }
    __syncthreads();
    T run = x - local + (w > 0 ? warp_tot[w - 1] : T(0));
    total = warp_tot[(nt >> 5) - 1];
    for (int i = lo; i < hi; ++i) {
        const T v = data[i];
        data[i] = run;
        run += v;
    }
    __syncthreads();
}

// One CTA of kMetaThreads threads.  Dynamic shared memory: C [nv] int64,
// pages [nv] int32, extra-split counts [nv] int32, begins [num_parts] int32 x 2.
constexpr int kMetaThreads = 256;

__global__ void __launch_bounds__(kMetaThreads) mla_metadata_kernel(const int32_t* seqlens, int const_len, int batch,
                                                                    int groups, int num_parts, int fixed_cost,
                                                                    int32_t* md, int32_t* num_splits)
{
    extern __shared__ __align__(16) uint8_t meta_smem[];
    grid_dependency_wait();
    grid_launch_dependents();  // the split-KV grid sets up while the schedule is computed
    __shared__ long long warp_tot_ll[32];
    __shared__ int warp_tot_i[32];
    const int nv = batch * groups;
    long long* C = reinterpret_cast<long long*>(meta_smem);
    int32_t* pages = reinterpret_cast<int32_t*>(C + nv);
    int32_t* extra = pages + nv;
    int32_t* begins = extra + nv;  // [num_parts][2]
    for (int v = threadIdx.x; v < nv; v += blockDim.x) {
        pages[v] = pages_of(seqlens ? seqlens[vb_request(v, batch)] : const_len);
        C[v] = pages[v] + fixed_cost;
        extra[v] = 0;
    }
    __syncthreads();
    long long total = 0;
    block_exclusive_scan(C, nv, warp_tot_ll, total);
    for (int p = threadIdx.x; p < num_parts; p += blockDim.x) {
        int32_t m[kMdInts];
        partition_range(p, num_parts, C, pages, nv, total, fixed_cost, m);
        begins[2 * p] = m[0];
        begins[2 * p + 1] = m[1];
        for (int i = 0; i < kMdInts; ++i) md[p * kMdInts + i] = m[i];
    }
    __syncthreads();
    for (int p = threadIdx.x; p < num_parts; p += blockDim.x) {
        const int bv = begins[2 * p], bb = begins[2 * p + 1];
        if (bb > 0) {
            int idx = 1;
            for (int q = p - 1; q >= 0 && begins[2 * q] == bv && begins[2 * q + 1] > 0; --q) ++idx;
            md[p * kMdInts + 4] = idx;
            atomicAdd(&extra[bv], 1);
        }
    }
    __syncthreads();
    for (int v = threadIdx.x; v < nv; v += blockDim.x) extra[v] += 1;  // splits of vb
    __syncthreads();
    int nsplit_total = 0;
    block_exclusive_scan(extra, nv, warp_tot_i, nsplit_total);
    for (int v = threadIdx.x; v < nv; v += blockDim.x) num_splits[v] = extra[v];
    if (threadIdx.x == 0) num_splits[nv] = nsplit_total;
}

static size_t metadata_smem_bytes(int nv, int num_parts)
{
    return static_cast<size_t>(nv) * (8 + 4 + 4) + static_cast<size_t>(num_parts) * 8 + 16;
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

static bool encode_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t cols, uint64_t rows,
                      uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw)
{
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool encode_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t d0, uint64_t d1,
                      uint64_t d2, uint64_t s1_bytes, uint64_t s2_bytes, uint32_t b0, uint32_t b1,
                      CUtensorMapSwizzle sw)
{
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1_bytes, s2_bytes};
    cuuint32_t box[3] = {b0, b1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launch configuration with programmatic stream serialization: the grid may start
// while the previous one in the stream finishes; each kernel calls
// grid_dependency_wait() before it reads global memory that grid could have written.
static void programmatic_launch(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attr, dim3 grid, dim3 block,
                                size_t smem, cudaStream_t stream)
{
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
}

// Heads [active_heads, h_q) are padding whose outputs nobody reads: a count that is not a
// multiple of 8 in (0, h_q], or an h_q that is not a multiple of 8, means every head (fail
// closed to the full computation, as the "FlashMLA vLLM Optimization" page's active-head
// switch does).
static int effective_active_heads(int active_heads, int h_q)
{
    return (active_heads > 0 && active_heads <= h_q && active_heads % 8 == 0 && h_q % 8 == 0) ? active_heads : h_q;
}

static size_t workspace_slots(int batch, int groups, int num_parts)
{
    return static_cast<size_t>(batch) * groups + static_cast<size_t>(num_parts);
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace layout: a control block of fixed size (the status word, then two int32 counters
// per virtual batch: split partials announced, combine CTAs past their wait), which must be
// zero before the first call and is left zero by every call that completes without a device
// error; then the split LSEs and the split partial outputs.  The control block's size does
// not depend on the problem, so calls of different sizes can share one workspace.
static void workspace_pointers(void* workspace, int batch, int groups, int num_parts, DecodeParams& prm)
{
    const size_t slots = workspace_slots(batch, groups, num_parts);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    prm.status = reinterpret_cast<int*>(ws);
    prm.ctl = reinterpret_cast<int*>(ws + kWorkspaceHeader);
    const size_t small = align_up(slots * kRowsPerGroup * sizeof(float), 256);  // one float per slot row
    prm.lse_accum = reinterpret_cast<float*>(ws + kControlBytes);
    prm.max_accum = reinterpret_cast<float*>(ws + kControlBytes + small);
    prm.o_accum = reinterpret_cast<float*>(ws + kControlBytes + 2 * small);
}

// Runs a per-device set-up step (a kernel attribute) once for each device it is used on,
// from any number of host threads.
struct PerDeviceOnce {
    static constexpr int kMaxDevices = 64;
    std::mutex m;
    std::atomic<bool> done[kMaxDevices] = {};

    template <typename F>
    cudaError_t run(F&& setup)
    {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMaxDevices) return setup();  // outside the table: every call
        if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
        std::lock_guard<std::mutex> lock(m);
        if (done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
        e = setup();
        if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
        return e;
    }
};

template <bool kRope, bool kFp16, bool kPadHeads, bool kFp8, bool kSparse>
static cudaError_t launch_splitkv(int grid, cudaStream_t stream, const CUtensorMap* maps, const DecodeParams& prm)
{
    auto kern = mla_splitkv_kernel<kRope, kFp16, kPadHeads, kFp8, kSparse>;
    const int smem = Layout<kRope, kFp8>::kSmemBytes;
    static PerDeviceOnce configured;  // the attribute is per device
    cudaError_t e = configured.run([&]() -> cudaError_t {
        cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (r != cudaSuccess) return r;
        if (kFp8) {
            // The warpgroups' register re-balancing hands out exactly what the launch holds
            // (128 per thread); with fewer at launch, setmaxnreg.inc would never return.
            cudaFuncAttributes fa;
            r = cudaFuncGetAttributes(&fa, kern);
            if (r != cudaSuccess) return r;
            if (fa.numRegs < static_cast<int>(kRegsLaunchFp8)) return cudaErrorInvalidConfiguration;
        }
        return cudaSuccess;
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    programmatic_launch(cfg, attr, dim3(grid), dim3(kFp8 ? kThreadsFp8 : kThreads), smem, stream);
    return cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], prm);
}

// The kernel variant with padding-head logic runs only when some heads are padding.
template <bool kRope, bool kFp16, bool kFp8 = false, bool kSparse = false>
static cudaError_t launch_splitkv_heads(int grid, cudaStream_t st, const CUtensorMap* maps, const DecodeParams& prm)
{
    return prm.active_heads < prm.h_q ? launch_splitkv<kRope, kFp16, true, kFp8, kSparse>(grid, st, maps, prm)
                                      : launch_splitkv<kRope, kFp16, false, kFp8, kSparse>(grid, st, maps, prm);
}

// The metadata kernel on `stream`: lengths from `seqlens`, or `const_len` for every request
// when `seqlens` is null (the sparse decode), at `fixed_cost` page units per chunk.
static mla_status launch_metadata(const int32_t* seqlens, int const_len, int batch, int heads_per_kv, int h_kv,
                                  int num_parts, int fixed_cost, int32_t* tile_md, int32_t* num_splits,
                                  void* stream)
{
    if (batch < 0 || heads_per_kv <= 0 || h_kv <= 0 || num_parts <= 0 || !tile_md || !num_splits)
        return MLA_ERR_INVALID_ARG;
    if (h_kv != 1) return MLA_ERR_UNSUPPORTED;
    const int nv = batch * row_groups(heads_per_kv);
    const size_t smem = metadata_smem_bytes(nv, num_parts);
    if (smem > 200 * 1024) return MLA_ERR_UNSUPPORTED;  // the schedule is built in one CTA's shared memory
    if (smem > 48 * 1024) {
        static PerDeviceOnce configured;
        if (configured.run([] {
                return cudaFuncSetAttribute(mla_metadata_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            200 * 1024);
            }) != cudaSuccess)
            return MLA_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    programmatic_launch(cfg, attr, dim3(1), dim3(kMetaThreads), smem, static_cast<cudaStream_t>(stream));
    const cudaError_t e = cudaLaunchKernelEx(&cfg, mla_metadata_kernel, seqlens, const_len, batch,
                                             row_groups(heads_per_kv), num_parts, fixed_cost, tile_md, num_splits);
    return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace mla

using namespace mla;

extern "C" {

const char* mla_status_string(int status)
{
    switch (status) {
        case MLA_OK: return "ok";
        case MLA_ERR_INVALID_ARG: return "invalid argument";
        case MLA_ERR_UNSUPPORTED: return "unsupported configuration";
        case MLA_ERR_WORKSPACE: return "workspace too small";
        case MLA_ERR_CUDA: return "CUDA error";
        case MLA_ERR_TIMEOUT: return "device pipeline wait timed out";
        case MLA_ERR_DEVICE_CHECK: return "block_table entry outside the cache";
        default: return "unknown status";
    }
}

mla_status mla_num_sm_parts(int device, int* num_parts)
{
    if (!num_parts) return MLA_ERR_INVALID_ARG;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || sms < 2) {
        cudaGetLastError();
        return MLA_ERR_CUDA;
    }
    *num_parts = sms / 2;
    return MLA_OK;
}

mla_status mla_metadata_sizes(int batch, int heads_per_kv, int h_kv, int num_parts, size_t* tile_md_ints,
                              size_t* num_splits_ints)
{
    if (!tile_md_ints || !num_splits_ints || batch < 0 || heads_per_kv <= 0 || h_kv <= 0 || num_parts <= 0)
        return MLA_ERR_INVALID_ARG;
    *tile_md_ints = static_cast<size_t>(num_parts) * kMdInts;
    *num_splits_ints = static_cast<size_t>(batch) * row_groups(heads_per_kv) + 1;
    return MLA_OK;
}

mla_status mla_get_metadata_host(const int32_t* cache_seqlens, int batch, int heads_per_kv, int h_kv,
                                 int num_parts, int is_fp8_kvcache, int32_t* tile_md, int32_t* num_splits)
{
    if (batch < 0 || heads_per_kv <= 0 || h_kv <= 0 || num_parts <= 0 || !tile_md || !num_splits ||
        (batch > 0 && !cache_seqlens))
        return MLA_ERR_INVALID_ARG;
    if (h_kv != 1) return MLA_ERR_UNSUPPORTED;
    for (int b = 0; b < batch; ++b)
        if (cache_seqlens[b] < 0) return MLA_ERR_INVALID_ARG;
    const int groups = row_groups(heads_per_kv);
    const size_t nv = static_cast<size_t>(batch) * groups;
    std::vector<long long> C(nv + 1);
    std::vector<int32_t> pages(nv + 1);
    schedule_host(cache_seqlens, batch, groups, num_parts, is_fp8_kvcache ? kFixedCostFp8 : kFixedCost, tile_md,
                  num_splits, C.data(), pages.data());
    return MLA_OK;
}

mla_status mla_get_metadata_sparse_host(int num_tokens, int topk, int h_q, int h_kv, int num_parts, int32_t* tile_md,
                                        int32_t* num_splits)
{
    if (num_tokens < 0 || topk < 0 || h_q <= 0 || h_kv <= 0 || h_q % h_kv || num_parts <= 0 || !tile_md ||
        !num_splits)
        return MLA_ERR_INVALID_ARG;
    if (h_kv != 1) return MLA_ERR_UNSUPPORTED;
    const int groups = row_groups(h_q / h_kv);
    const size_t nv = static_cast<size_t>(num_tokens) * groups;
    std::vector<int32_t> lens(static_cast<size_t>(num_tokens) + 1, topk);
    std::vector<long long> C(nv + 1);
    std::vector<int32_t> pages(nv + 1);
    schedule_host(lens.data(), num_tokens, groups, num_parts, kFixedCostSparse, tile_md, num_splits, C.data(),
                  pages.data());
    return MLA_OK;
}

mla_status mla_get_metadata(const int32_t* cache_seqlens, int batch, int heads_per_kv, int h_kv, int num_parts,
                            int is_fp8_kvcache, int32_t* tile_md, int32_t* num_splits, void* stream)
{
    if (batch > 0 && !cache_seqlens) return MLA_ERR_INVALID_ARG;
    return launch_metadata(cache_seqlens, 0, batch, heads_per_kv, h_kv, num_parts,
                           is_fp8_kvcache ? kFixedCostFp8 : kFixedCost, tile_md, num_splits, stream);
}

mla_status mla_get_metadata_sparse(int num_tokens, int topk, int h_q, int h_kv, int num_parts, int32_t* tile_md,
                                   int32_t* num_splits, void* stream)
{
    if (topk < 0 || h_kv <= 0 || h_q % h_kv) return MLA_ERR_INVALID_ARG;
    return launch_metadata(nullptr, topk, num_tokens, h_q / h_kv, h_kv, num_parts, kFixedCostSparse, tile_md,
                           num_splits, stream);
}

size_t mla_decode_workspace_zero_bytes(int batch, int s_q, int h_q, int h_kv)
{
    if (batch < 0 || s_q <= 0 || h_q <= 0 || h_kv <= 0 || h_q % h_kv) return 0;
    return kControlBytes;
}

size_t mla_decode_workspace_bytes(int batch, int s_q, int h_q, int h_kv, int num_parts)
{
    if (batch < 0 || s_q <= 0 || h_q <= 0 || h_kv <= 0 || num_parts <= 0 || h_q % h_kv) return 0;
    const int groups = row_groups(s_q * h_q / h_kv);
    if (static_cast<long long>(batch) * groups > kMaxVirtualBatches) return 0;
    const size_t slots = workspace_slots(batch, groups, num_parts);
    size_t bytes = kControlBytes;
    bytes += 2 * align_up(slots * kRowsPerGroup * sizeof(float), 256);  // split LSEs and maxima
    bytes += slots * kRowsPerGroup * kDv * sizeof(float);
    return bytes;
}

// Validates the arguments and fills the kernel parameters and tensor maps.
static mla_status prepare_decode(const void* q, int batch, int s_q, int h_q, int d_qk, const void* kvcache,
                                 int num_blocks, int page_size, int h_kv, const int32_t* block_table,
                                 int max_blocks_per_seq, const int32_t* cache_seqlens, int dv, int dtype,
                                 const int32_t* tile_md, int num_parts, const int32_t* num_splits, int causal,
                                 float softmax_scale, int active_heads, void* o, float* lse, void* workspace,
                                 size_t workspace_bytes, const int32_t* indices, int topk, DecodeParams& prm,
                                 CUtensorMap* maps, long long cache_rows_override = 0)
{
    // indices != null: the sparse decode, with batch = requests x query tokens and s_q = 1;
    // no block table, no sequence lengths, no causal mask
    const bool sparse = indices != nullptr;
    if (batch < 0 || s_q <= 0 || h_q <= 0 || h_kv <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 ||
        num_parts <= 0 || (causal != 0 && causal != 1) || topk < 0)
        return MLA_ERR_INVALID_ARG;
    if (dtype != MLA_BF16 && dtype != MLA_FP16 && dtype != MLA_BF16_FP8KV) return MLA_ERR_INVALID_ARG;
    if (page_size != kPage || h_kv != 1 || (d_qk != 576 && d_qk != 512) || dv != kDv) return MLA_ERR_UNSUPPORTED;
    if (dtype == MLA_BF16_FP8KV && d_qk != 576) return MLA_ERR_UNSUPPORTED;  // the FP8 row carries 64 RoPE values
    if (sparse && d_qk != 576) return MLA_ERR_UNSUPPORTED;  // the sparse kernels are built for 576-wide rows
    if (batch > 0 && (!q || !kvcache || (!sparse && (!block_table || !cache_seqlens)) || !tile_md || !num_splits ||
                      !o || !lse || !workspace))
        return MLA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(kvcache) & 15) ||
        (reinterpret_cast<uintptr_t>(o) & 15) || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return MLA_ERR_INVALID_ARG;
    const int rows = s_q * h_q;
    const int groups = row_groups(rows);
    if (static_cast<long long>(batch) * groups > kMaxVirtualBatches) return MLA_ERR_UNSUPPORTED;
    const size_t need = mla_decode_workspace_bytes(batch, s_q, h_q, h_kv, num_parts);
    if (batch > 0 && workspace_bytes < need) return MLA_ERR_WORKSPACE;
    if (static_cast<long long>(num_blocks) * kPage >= (1ll << 31)) return MLA_ERR_UNSUPPORTED;
    // rows of the cache the sparse gathers address: every page's rows, or a flat kv's own count
    const long long cache_rows = cache_rows_override > 0 ? cache_rows_override : static_cast<long long>(num_blocks) * kPage;
    if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt(static_cast<float>(d_qk));
    prm = DecodeParams{};
    prm.block_table = sparse ? nullptr : block_table;
    prm.seqlens = sparse ? nullptr : cache_seqlens;
    prm.indices = indices;
    prm.topk = topk;
    prm.cache_rows = static_cast<int>(cache_rows);
    prm.md = tile_md;
    prm.num_splits = num_splits;
    prm.q = q;
    prm.kvcache = kvcache;
    prm.o = o;
    prm.lse = lse;
    prm.batch = batch;
    prm.s_q = s_q;
    prm.h_q = h_q;
    prm.rows = rows;
    prm.groups = groups;
    prm.max_blocks = max_blocks_per_seq;
    prm.num_blocks = num_blocks;
    prm.causal = sparse ? 0 : causal;
    prm.box_rows = rows < 64 ? rows : 64;  // query rows per CTA of the pair
    prm.scale_log2 = softmax_scale * 1.4426950408889634f;
    prm.active_heads = effective_active_heads(active_heads, h_q);
    prm.o_align32 = (reinterpret_cast<uintptr_t>(o) & 31) == 0;
    prm.dtype = dtype;
    prm.d_qk = d_qk;
    prm.num_parts = num_parts;
    if (batch == 0) return MLA_OK;
    workspace_pointers(workspace, batch, groups, num_parts, prm);
    if (!maps) return MLA_OK;

    const CUtensorMapDataType dt =
        dtype == MLA_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const uint64_t row_bytes = static_cast<uint64_t>(d_qk) * 2;
    const uint64_t kv_rows = static_cast<uint64_t>(cache_rows);
    // Q: [batch][rows][d_qk], box 64 columns x (up to) 64 rows;
    // K: cache rows, box 64 columns x 32 tokens (half a page, one CTA's share);
    // V: cache rows, box 64 columns x 64 tokens (a page).
    // FP8 cache: rows of 656 bytes; K: boxes of 128 bytes x 32 rows (latent slices), V: boxes
    // of 16 bytes x 32 rows (the scales), no swizzle.
    const bool fp8 = dtype == MLA_BF16_FP8KV;
    if (sparse && !fp8) {
        // 16-bit sparse: K and V gathered row by row (tile::gather4, one-row boxes of 64 columns);
        // the maps end at the last row, so an invalid entry's row (cache_rows) reads zeros
        const bool ok_g =
            encode_3d(&maps[0], q, dt, d_qk, rows, batch, row_bytes, row_bytes * rows, 64, prm.box_rows,
                      CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_2d(&maps[1], kvcache, dt, d_qk, kv_rows, row_bytes, 64, 1, CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_2d(&maps[2], kvcache, dt, d_qk, kv_rows, row_bytes, 64, 1, CU_TENSOR_MAP_SWIZZLE_128B);
        return ok_g ? MLA_OK : MLA_ERR_CUDA;
    }
    const bool ok =
        encode_3d(&maps[0], q, dt, d_qk, rows, batch, row_bytes, row_bytes * rows, 64, prm.box_rows,
                  CU_TENSOR_MAP_SWIZZLE_128B) &&
        (fp8 ? encode_2d(&maps[1], kvcache, CU_TENSOR_MAP_DATA_TYPE_UINT8, kFp8Row, kv_rows, kFp8Row, 128,
                         kPage / 2, CU_TENSOR_MAP_SWIZZLE_NONE)
             : encode_2d(&maps[1], kvcache, dt, d_qk, kv_rows, row_bytes, 64, kPage / 2,
                         CU_TENSOR_MAP_SWIZZLE_128B)) &&
        (fp8 ? encode_2d(&maps[2], kvcache, CU_TENSOR_MAP_DATA_TYPE_UINT8, kFp8Row, kv_rows, kFp8Row, 16,
                         kPage / 2, CU_TENSOR_MAP_SWIZZLE_NONE)
             : encode_2d(&maps[2], kvcache, dt, d_qk, kv_rows, row_bytes, 64, kPage, CU_TENSOR_MAP_SWIZZLE_128B));
    return ok ? MLA_OK : MLA_ERR_CUDA;
}

static mla_status launch_splitkv_stage(const DecodeParams& prm, const CUtensorMap* maps, cudaStream_t st)
{
    const int grid = 2 * prm.num_parts;
    cudaError_t e;
    if (prm.indices && prm.dtype == MLA_BF16_FP8KV)
        e = launch_splitkv_heads<true, false, true, true>(grid, st, maps, prm);
    else if (prm.indices)
        e = prm.dtype == MLA_FP16 ? launch_splitkv_heads<true, true, false, true>(grid, st, maps, prm)
                                  : launch_splitkv_heads<true, false, false, true>(grid, st, maps, prm);
    else if (prm.dtype == MLA_BF16_FP8KV)
        e = launch_splitkv_heads<true, false, true>(grid, st, maps, prm);
    else if (prm.d_qk == 576)
        e = prm.dtype == MLA_FP16 ? launch_splitkv_heads<true, true>(grid, st, maps, prm)
                                  : launch_splitkv_heads<true, false>(grid, st, maps, prm);
    else
        e = prm.dtype == MLA_FP16 ? launch_splitkv_heads<false, true>(grid, st, maps, prm)
                                  : launch_splitkv_heads<false, false>(grid, st, maps, prm);
    return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

static mla_status launch_combine_stage(const DecodeParams& prm, cudaStream_t st)
{
    const int rows_max = prm.rows < kRowsPerGroup ? prm.rows : kRowsPerGroup;
    // Fewer than one virtual batch per 4 partitions means many splits per virtual batch
    // (long sequences): read each row's splits in parallel.
    const long long nv = static_cast<long long>(prm.batch) * prm.groups;
    const bool split_parallel = 4 * nv < prm.num_parts;
    dim3 cgrid(static_cast<unsigned>(nv), split_parallel ? rows_max : (rows_max + 3) / 4);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    programmatic_launch(cfg, attr, cgrid, dim3(128), 0, st);
    cudaError_t e;
    if (prm.dtype == MLA_FP16)
        e = split_parallel ? cudaLaunchKernelEx(&cfg, mla_combine_kernel<true, true>, prm)
                           : cudaLaunchKernelEx(&cfg, mla_combine_kernel<true, false>, prm);
    else
        e = split_parallel ? cudaLaunchKernelEx(&cfg, mla_combine_kernel<false, true>, prm)
                           : cudaLaunchKernelEx(&cfg, mla_combine_kernel<false, false>, prm);
    return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

#define MLA_DECODE_ARGS                                                                                          \
    q, batch, s_q, h_q, d_qk, kvcache, num_blocks, page_size, h_kv, block_table, max_blocks_per_seq,            \
        cache_seqlens, dv, dtype, tile_md, num_parts, num_splits, causal, softmax_scale, active_heads, o, lse,   \
        workspace, workspace_bytes, nullptr, 0

mla_status mla_decode_with_kvcache(const void* q, int batch, int s_q, int h_q, int d_qk, const void* kvcache,
                                   int num_blocks, int page_size, int h_kv, const int32_t* block_table,
                                   int max_blocks_per_seq, const int32_t* cache_seqlens, int dv, int dtype,
                                   const int32_t* tile_md, int num_parts, const int32_t* num_splits, int causal,
                                   float softmax_scale, int active_heads, void* o, float* lse, void* workspace,
                                   size_t workspace_bytes, void* stream)
{
    DecodeParams prm;
    CUtensorMap maps[kNumMaps];
    mla_status s = prepare_decode(MLA_DECODE_ARGS, prm, maps);
    if (s != MLA_OK || batch == 0) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = launch_splitkv_stage(prm, maps, st);
    if (s != MLA_OK) return s;
    return launch_combine_stage(prm, st);
}

mla_status mla_decode_splitkv(const void* q, int batch, int s_q, int h_q, int d_qk, const void* kvcache,
                              int num_blocks, int page_size, int h_kv, const int32_t* block_table,
                              int max_blocks_per_seq, const int32_t* cache_seqlens, int dv, int dtype,
                              const int32_t* tile_md, int num_parts, const int32_t* num_splits, int causal,
                              float softmax_scale, int active_heads, void* o, float* lse, void* workspace,
                              size_t workspace_bytes, void* stream)
{
    DecodeParams prm;
    CUtensorMap maps[kNumMaps];
    mla_status s = prepare_decode(MLA_DECODE_ARGS, prm, maps);
    if (s != MLA_OK || batch == 0) return s;
    return launch_splitkv_stage(prm, maps, static_cast<cudaStream_t>(stream));
}

mla_status mla_decode_combine(int batch, int s_q, int h_q, int h_kv, int dv, int dtype, const int32_t* num_splits,
                              int num_parts, int active_heads, void* o, float* lse, void* workspace,
                              size_t workspace_bytes, void* stream)
{
    if (batch < 0 || s_q <= 0 || h_q <= 0 || h_kv <= 0 || num_parts <= 0) return MLA_ERR_INVALID_ARG;
    if (dtype != MLA_BF16 && dtype != MLA_FP16 && dtype != MLA_BF16_FP8KV) return MLA_ERR_INVALID_ARG;
    if (h_kv != 1 || dv != kDv) return MLA_ERR_UNSUPPORTED;
    if (static_cast<long long>(batch) * row_groups(s_q * h_q) > kMaxVirtualBatches) return MLA_ERR_UNSUPPORTED;
    if (batch == 0) return MLA_OK;
    if (!num_splits || !o || !lse || !workspace) return MLA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return MLA_ERR_INVALID_ARG;
    if (workspace_bytes < mla_decode_workspace_bytes(batch, s_q, h_q, h_kv, num_parts)) return MLA_ERR_WORKSPACE;
    const int rows = s_q * h_q;
    const int groups = row_groups(rows);
    DecodeParams prm{};
    prm.num_splits = num_splits;
    prm.o = o;
    prm.lse = lse;
    prm.rows = rows;
    prm.groups = groups;
    prm.batch = batch;
    prm.dtype = dtype;
    prm.num_parts = num_parts;
    prm.h_q = h_q;
    prm.active_heads = effective_active_heads(active_heads, h_q);
    workspace_pointers(workspace, batch, groups, num_parts, prm);
    return launch_combine_stage(prm, static_cast<cudaStream_t>(stream));
}

#ifdef MLA_TIMELINE
// Timeline build only: copies the event array (kTlMaxCtas x kTlCtaWords words) to `host`.
MLA_API mla_status mla_timeline_read(uint32_t* host, size_t words)
{
    if (!host || words < static_cast<size_t>(kTlMaxCtas) * kTlCtaWords) return MLA_ERR_INVALID_ARG;
    return cudaMemcpyFromSymbol(host, g_timeline, sizeof(g_timeline)) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
#endif

}  // extern "C"

// The sparse decode: the split-KV stage, then (unless `only_splitkv`) the combine stage.
static mla_status decode_sparse(const void* q, int batch, int s_q, int h_q, int d_qk, const void* kvcache,
                                int num_blocks, int page_size, int h_kv, const int32_t* indices, int topk, int dv,
                                int dtype, const int32_t* tile_md, int num_parts, const int32_t* num_splits,
                                float softmax_scale, int active_heads, void* o, float* lse, void* workspace,
                                size_t workspace_bytes, void* stream, bool only_splitkv)
{
    if (batch < 0 || s_q <= 0 || topk < 0) return MLA_ERR_INVALID_ARG;
    if (batch > 0 && !indices) return MLA_ERR_INVALID_ARG;
    if (static_cast<long long>(batch) * s_q > (1ll << 30)) return MLA_ERR_UNSUPPORTED;
    DecodeParams prm;
    CUtensorMap maps[kNumMaps];
    // every query token is a request of its own: batch * s_q requests of one token
    const int tokens = batch * s_q;
    const int32_t* one = indices ? indices : reinterpret_cast<const int32_t*>(&prm);  // not read when batch == 0
    mla_status s = prepare_decode(q, tokens, 1, h_q, d_qk, kvcache, num_blocks, page_size, h_kv, nullptr, 1,
                                  nullptr, dv, dtype, tile_md, num_parts, num_splits, 0, softmax_scale, active_heads,
                                  o, lse, workspace, workspace_bytes, one, topk, prm, maps);
    if (s != MLA_OK || tokens == 0) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = launch_splitkv_stage(prm, maps, st);
    if (s != MLA_OK || only_splitkv) return s;
    return launch_combine_stage(prm, st);
}

extern "C" {

mla_status mla_decode_sparse(const void* q, int batch, int s_q, int h_q, int d_qk, const void* kvcache, int num_blocks,
                             int page_size, int h_kv, const int32_t* indices, int topk, int dv, int dtype,
                             const int32_t* tile_md, int num_parts, const int32_t* num_splits, float softmax_scale,
                             int active_heads, void* o, float* lse, void* workspace, size_t workspace_bytes,
                             void* stream)
{
    return decode_sparse(q, batch, s_q, h_q, d_qk, kvcache, num_blocks, page_size, h_kv, indices, topk, dv, dtype,
                         tile_md, num_parts, num_splits, softmax_scale, active_heads, o, lse, workspace,
                         workspace_bytes, stream, false);
}

mla_status mla_decode_sparse_splitkv(const void* q, int batch, int s_q, int h_q, int d_qk, const void* kvcache,
                                     int num_blocks, int page_size, int h_kv, const int32_t* indices, int topk,
                                     int dv, int dtype, const int32_t* tile_md, int num_parts,
                                     const int32_t* num_splits, float softmax_scale, int active_heads, void* o,
                                     float* lse, void* workspace, size_t workspace_bytes, void* stream)
{
    return decode_sparse(q, batch, s_q, h_q, d_qk, kvcache, num_blocks, page_size, h_kv, indices, topk, dv, dtype,
                         tile_md, num_parts, num_splits, softmax_scale, active_heads, o, lse, workspace,
                         workspace_bytes, stream, true);
}

mla_status mla_sparse_prefill(const void* q, int s_q, int h_q, int d_qk, const void* kv, int s_kv, int h_kv,
                              const int32_t* indices, int topk, int dv, int dtype, float sm_scale, const int32_t* tile_md,
                              int num_parts, const int32_t* num_splits, void* out, float* max_logits, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream)
{
    if (s_q < 0 || s_kv <= 0 || topk < 0 || (s_q > 0 && (!indices || !max_logits))) return MLA_ERR_INVALID_ARG;
    if (dtype != MLA_BF16 && dtype != MLA_FP16) return dtype == MLA_BF16_FP8KV ? MLA_ERR_UNSUPPORTED : MLA_ERR_INVALID_ARG;
    DecodeParams prm;
    CUtensorMap maps[kNumMaps];
    // every query token is a request; the kv rows are addressed directly (no pages, no table)
    const int pages = (s_kv + kPage - 1) / kPage;
    const int32_t* one = indices ? indices : reinterpret_cast<const int32_t*>(&prm);  // not read when s_q == 0
    mla_status s = prepare_decode(q, s_q, 1, h_q, d_qk, kv, pages, kPage, h_kv, nullptr, 1, nullptr, dv, dtype, tile_md,
                                  num_parts, num_splits, 0, sm_scale, 0, out, lse, workspace, workspace_bytes, one,
                                  topk, prm, maps, s_kv);
    if (s != MLA_OK || s_q == 0) return s;
    prm.max_logits = max_logits;
    prm.lse_base2 = 1;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = launch_splitkv_stage(prm, maps, st);
    if (s != MLA_OK) return s;
    return launch_combine_stage(prm, st);
}

mla_status mla_read_device_status(void* workspace, int clear, int* device_status, void* stream)
{
    if (!workspace || !device_status) return MLA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int v = 0;
    if (cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return MLA_ERR_CUDA;
    *device_status = v;
    // the whole control block: after a device error its counters may be left nonzero too
    if (clear && cudaMemsetAsync(workspace, 0, kControlBytes, st) != cudaSuccess) return MLA_ERR_CUDA;
    return MLA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ allocation-free decode
// Scratch of mla_decode_with_kvcache_noalloc: the same layout as a caller-provided
// workspace (status header, split LSEs, split partial outputs), held in a
// file-scope device array of MLA_NOALLOC_SCRATCH_BYTES on every GPU that loads
// this library, for the life of the process.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};  // device address of the array, per device

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address comes from the
// runtime, once per device, with that device current.
mla_status noalloc_scratch(void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return MLA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
            cudaGetLastError();
            return MLA_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
    return MLA_OK;
}
}  // namespace

extern "C" mla_status mla_decode_with_kvcache_noalloc(const void* q, int batch, int s_q, int h_q, int d_qk,
                                                      const void* kvcache, int num_blocks, int page_size, int h_kv,
                                                      const int32_t* block_table, int max_blocks_per_seq,
                                                      const int32_t* cache_seqlens, int dv, int dtype,
                                                      const int32_t* tile_md, int num_parts,
                                                      const int32_t* num_splits, int causal, float softmax_scale,
                                                      int active_heads, void* o, float* lse, void* stream)
{
    if (batch < 0 || s_q <= 0 || h_q <= 0 || h_kv <= 0 || num_parts <= 0) return MLA_ERR_INVALID_ARG;
    if (batch == 0) return MLA_OK;
    const size_t need = mla_decode_workspace_bytes(batch, s_q, h_q, h_kv, num_parts);
    if (need == 0) return MLA_ERR_INVALID_ARG;
    if (need > MLA_NOALLOC_SCRATCH_BYTES) return MLA_ERR_WORKSPACE;  // problem too large for the fixed scratch
    void* scratch = nullptr;
    mla_status st = noalloc_scratch(&scratch);
    if (st != MLA_OK) return st;
    // The status word and this call's split / combine counters must start at zero (a call
    // that met a device error may have left them nonzero); the split partials are always
    // written before they are read, so the rest of the scratch needs no clearing.
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const size_t nv = static_cast<size_t>(batch) * row_groups(s_q * h_q / h_kv);
    if (cudaMemsetAsync(scratch, 0, kWorkspaceHeader + 2 * sizeof(int32_t) * nv, cs) != cudaSuccess)
        return MLA_ERR_CUDA;
    return mla_decode_with_kvcache(q, batch, s_q, h_q, d_qk, kvcache, num_blocks, page_size, h_kv, block_table,
                                   max_blocks_per_seq, cache_seqlens, dv, dtype, tile_md, num_parts, num_splits,
                                   causal, softmax_scale, active_heads, o, lse, scratch, MLA_NOALLOC_SCRATCH_BYTES,
                                   stream);
}

extern "C" mla_status mla_read_noalloc_status(int clear, int* device_status, void* stream)
{
    if (!device_status) return MLA_ERR_INVALID_ARG;
    void* scratch = nullptr;
    mla_status st = noalloc_scratch(&scratch);
    if (st != MLA_OK) return st;
    return mla_read_device_status(scratch, clear, device_status, stream);
}
