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
// * One two-CTA cluster (two SMs) per scheduler partition.  The 128 query rows
//   of a row group are the MMA M dimension in both CTAs.  The d_qk columns are
//   split between the CTAs: CTA c owns latent columns [256c, 256c+256) and
//   RoPE columns [512 + 32c, 512 + 32c + 32).  Each CTA loads only its columns
//   of Q and of every cached page (every KV byte is read from HBM once, by one
//   CTA), computes the partial logits S_c = Q_c K_c^T with tcgen05 into tensor
//   memory, and the two partials are summed by exchanging them through
//   distributed shared memory (st.async into the peer's buffer).  Both CTAs
//   then hold the same logits and run the same online softmax, so each can
//   accumulate its half of O = P V (V columns [256c, 256c+256)) in its own
//   tensor memory: O half (256 columns) + two S/P buffers (2 x 64) = 384 of
//   the 512 TMEM columns.
// * Warp roles per CTA: warps 0-3 softmax / correction / epilogue (thread =
//   query row = TMEM lane), warp 4 TMA producer (Q per chunk, one 64-token page
//   per pipeline stage, pages found through the block table), warp 5 MMA issuer.
// * P is written back into the S buffer in tensor memory (16-bit, two per
//   column) and is the A operand of the PV MMA; V is read from the same shared
//   memory stage as K (MN-major descriptor), never loaded twice.
// * Online softmax in base 2 with a lazily moved reference maximum: O is only
//   rescaled when the running maximum grows by more than 2^8.
// * Split chunks write fp32 partial O and LSE to the workspace; the combine
//   kernel merges them.
//
// Every mbarrier wait is bounded: after kWaitTimeoutNs the waiting thread sets
// an abort flag (seen by both CTAs of the cluster) and MLA_ERR_TIMEOUT in the
// workspace status word, and every role winds down and frees tensor memory.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/mla_decode.h"
#include "ptx.cuh"
#include "scheduler.cuh"

namespace mla {

constexpr int kThreads = 192;          // 4 softmax warps + TMA warp + MMA warp
constexpr int kTmaWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kDv = 512;
constexpr int kDvHalf = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;         // O half: columns [0, 256)
constexpr uint32_t kTmemS = 256;       // S/P buffers: [256, 320), [320, 384)
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;
constexpr int kWorkspaceHeader = 256;

template <bool kRope>
struct Layout {
    static constexpr int kBoxes = 4;                                   // 64-column SW128 boxes per CTA
    static constexpr int kQBytes = kBoxes * 16384 + (kRope ? 8192 : 0);   // 128 rows
    static constexpr int kStageBytes = kBoxes * 8192 + (kRope ? 4096 : 0);  // 64 tokens
    static constexpr int kStages = kRope ? 3 : 4;
    static constexpr int kXBytes = 128 * 64 * 4;                       // peer partial logits
    static constexpr int kKSlices = kBoxes * 4 + (kRope ? 2 : 0);      // K=16 MMA steps for S
    static constexpr int kOffQ = 0;
    static constexpr int kOffKV = kOffQ + kQBytes;
    static constexpr int kOffX = kOffKV + kStages * kStageBytes;
    static constexpr int kOffBar = kOffX + kXBytes;
    static constexpr int kBarBytes = 512;
    static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;      // + alignment slack
};

// Barrier slots (8 bytes each) inside the barrier area.
enum BarSlot : int {
    kBarQFull = 0,
    kBarQFree = 1,
    kBarSFull = 2,    // 2 slots
    kBarPFull = 4,
    kBarPvDone = 5,
    kBarOFull = 6,
    kBarOFree = 7,
    kBarDrain = 8,
    kBarXFull = 9,    // 4 slots
    kBarXFree = 13,   // 4 slots
    kBarKvFull = 17,  // kStages slots
    kBarKvEmpty = 21, // kStages slots
    kBarCount = 25
};
constexpr int kOffTmemSlot = kBarCount * 8;       // uint32 written by tcgen05.alloc
constexpr int kOffAbort = kOffTmemSlot + 4;       // int abort flag

struct DecodeParams {
    const int32_t* block_table;
    const int32_t* seqlens;
    const int32_t* md;
    const int32_t* num_splits;
    void* o;
    float* lse;
    float* o_accum;     // [slots, 128, 512]
    float* lse_accum;   // [slots, 128]
    int* status;
    int batch, s_q, h_q, rows, groups, max_blocks, num_blocks, causal, box_rows;
    float scale_log2;
    int dtype, d_qk, num_parts;  // host-side dispatch only
};

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
        if (mbar_try_wait(bar, parity)) return true;
        const uint64_t t0 = global_timer_ns();
        while (true) {
            for (int i = 0; i < 32; ++i)
                if (mbar_try_wait(bar, parity)) return true;
            if (aborted()) return false;
            if (global_timer_ns() - t0 > kWaitTimeoutNs) {
                raise(MLA_ERR_TIMEOUT);
                return false;
            }
        }
    }
};

// Iterates the chunks (vb, blk_lo, blk_hi) of one scheduler partition.
struct ChunkIter {
    int vb, blk, end_vb, end_blk, groups;
    const int32_t* seqlens;

    __device__ bool next(int& out_vb, int& lo, int& hi)
    {
        if (!(vb < end_vb || (vb == end_vb && blk < end_blk))) return false;
        const int n = pages_of(seqlens[vb / groups]);
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

// ------------------------------------------------------------------ split-KV kernel
template <bool kRope, bool kFp16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    mla_splitkv_kernel(const __grid_constant__ CUtensorMap tm_q128, const __grid_constant__ CUtensorMap tm_q64,
                       const __grid_constant__ CUtensorMap tm_kv128, const __grid_constant__ CUtensorMap tm_kv64,
                       const DecodeParams p)
{
    using L = Layout<kRope>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_addr(smem);
    const uint32_t s_q = s_base + L::kOffQ;
    const uint32_t s_kv = s_base + L::kOffKV;
    const uint32_t s_x = s_base + L::kOffX;
    const uint32_t s_bar = s_base + L::kOffBar;
    auto bar = [&](int slot) { return s_bar + 8u * slot; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t cta = cluster_cta_rank();
    const uint32_t peer = cta ^ 1u;
    const int part = blockIdx.x >> 1;

    // ---------------- set-up
    if (threadIdx.x == 0) {
        mbar_init(bar(kBarQFull), 1);
        mbar_init(bar(kBarQFree), 1);
        mbar_init(bar(kBarSFull + 0), 1);
        mbar_init(bar(kBarSFull + 1), 1);
        mbar_init(bar(kBarPFull), 4);
        mbar_init(bar(kBarPvDone), 1);
        mbar_init(bar(kBarOFull), 1);
        mbar_init(bar(kBarOFree), 4);
        mbar_init(bar(kBarDrain), 1);
        for (int w = 0; w < 4; ++w) {
            mbar_init(bar(kBarXFull + w), 1);
            mbar_init(bar(kBarXFree + w), 32);
        }
        for (int s = 0; s < L::kStages; ++s) {
            mbar_init(bar(kBarKvFull + s), 1);
            mbar_init(bar(kBarKvEmpty + s), 1);
        }
        *reinterpret_cast<volatile int*>(smem + L::kOffBar + kOffAbort) = 0;
        fence_mbar_init();
    }
    // Query rows beyond the loaded box stay zero (finite) for the whole kernel.
    if (p.box_rows < kRowsPerGroup) {
        uint4* q4 = reinterpret_cast<uint4*>(smem + L::kOffQ);
        for (int i = threadIdx.x; i < L::kQBytes / 16; i += kThreads) q4[i] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(s_bar + kOffTmemSlot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == kTmaWarp && lane == 0) {
        prefetch_tensormap(&tm_q128);
        prefetch_tensormap(&tm_kv128);
        if (kRope) {
            prefetch_tensormap(&tm_q64);
            prefetch_tensormap(&tm_kv64);
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // peer barriers initialised before any remote arrive / store
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kOffBar + kOffTmemSlot);

    Sync sync{s_bar + kOffAbort, map_to_cta(s_bar + kOffAbort, peer), p.status};
    const int32_t* md = p.md + part * kMdInts;
    ChunkIter chunks{md[0], md[1], md[2], md[3], p.groups, p.seqlens};
    const int begin_vb = md[0];
    const int begin_split = md[4];
    const uint32_t col0 = 256u * cta;          // first latent column of this CTA
    const uint32_t rope_col = 512u + 32u * cta;

    if (warp == kTmaWarp) {
        // ============================ TMA producer ============================
        if (lane == 0) {
            uint32_t g = 0, k = 0;
            int vb, lo, hi;
            bool ok = true;
            bool q_issued = false;
            const uint32_t q_tx = p.box_rows * (L::kBoxes * 128 + (kRope ? 64 : 0));
            while (ok && chunks.next(vb, lo, hi)) {
                if (hi <= lo) continue;
                const int b = vb / p.groups, rg = vb % p.groups;
                if (!(ok = sync.wait(bar(kBarQFree), (k & 1) ^ 1))) break;
                mbar_arrive_expect_tx(bar(kBarQFull), q_tx);
                q_issued = true;
                for (int i = 0; i < L::kBoxes; ++i)
                    tma_load_3d(s_q + i * 16384, &tm_q128, bar(kBarQFull), col0 + 64 * i, rg * kRowsPerGroup, b);
                if (kRope)
                    tma_load_3d(s_q + L::kBoxes * 16384, &tm_q64, bar(kBarQFull), rope_col, rg * kRowsPerGroup, b);
                const int32_t* table = p.block_table + static_cast<size_t>(b) * p.max_blocks;
                for (int blk = lo; blk < hi; ++blk, ++g) {
                    const uint32_t st = g % L::kStages;
                    if (!(ok = sync.wait(bar(kBarKvEmpty + st), ((g / L::kStages) & 1) ^ 1))) break;
                    int page = blk < p.max_blocks ? __ldg(table + blk) : -1;
                    if (page < 0 || page >= p.num_blocks) {
                        atomicCAS(p.status, 0, MLA_ERR_DEVICE_CHECK);
                        page = 0;  // keep the pipeline in bounds; the status word reports the error
                    }
                    const uint32_t dst = s_kv + st * L::kStageBytes;
                    mbar_arrive_expect_tx(bar(kBarKvFull + st), L::kStageBytes);
                    for (int i = 0; i < L::kBoxes; ++i)
                        tma_load_2d(dst + i * 8192, &tm_kv128, bar(kBarKvFull + st), col0 + 64 * i, page * kPage);
                    if (kRope)
                        tma_load_2d(dst + L::kBoxes * 8192, &tm_kv64, bar(kBarKvFull + st), rope_col, page * kPage);
                }
                ++k;
            }
            if (!ok) {
                // Let the loads already issued land before shared memory goes away:
                // the most recent load into each stage, and the last Q load.
                const uint64_t t0 = global_timer_ns();
                for (uint32_t i = 0; i < L::kStages && i < g; ++i) {
                    const uint32_t gl = g - 1 - i;
                    while (!mbar_try_wait(bar(kBarKvFull + gl % L::kStages), (gl / L::kStages) & 1) &&
                           global_timer_ns() - t0 < 100000000ull) {
                    }
                }
                if (q_issued) {
                    const uint32_t kl = k;  // chunk whose Q was issued last
                    while (!mbar_try_wait(bar(kBarQFull), kl & 1) && global_timer_ns() - t0 < 100000000ull) {
                    }
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ============================ MMA issuer ============================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = instr_desc_f16(kFp16, 128, 64, false);
            constexpr uint32_t idesc_pv = instr_desc_f16(kFp16, 128, 256, true);
            uint32_t g = 0, k = 0;
            int vb, lo, hi;
            bool ok = true;
            auto issue_pv = [&](uint32_t gp, bool first) -> bool {
                if (!sync.wait(bar(kBarPFull), gp & 1)) return false;
                if (first && !sync.wait(bar(kBarOFree), (k & 1) ^ 1)) return false;
                tc_fence_after();
                const uint32_t st = gp % L::kStages;
                const uint32_t p_tmem = tmem + kTmemS + 64 * (gp & 1);
                const uint32_t v_base = s_kv + st * L::kStageBytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    // B = V[16 tokens, 256 columns], MN-major SW128: 64-column groups 8 KB apart
                    // (LBO), 8-token groups 1 KB apart (SBO).
                    const uint64_t vdesc = smem_desc(v_base + kk * 2048, 8192, 1024, kLayoutSW128);
                    mma_ts(tmem + kTmemO, p_tmem + 8 * kk, vdesc, idesc_pv, (first && kk == 0) ? 0u : 1u);
                }
                mma_commit(bar(kBarKvEmpty + st));
                mma_commit(bar(kBarPvDone));
                return true;
            };
            while (ok && chunks.next(vb, lo, hi)) {
                const int n = hi - lo;
                if (n <= 0) continue;
                if (!(ok = sync.wait(bar(kBarQFull), k & 1))) break;
                tc_fence_after();
                for (int j = 0; j < n && ok; ++j) {
                    const uint32_t gp = g + j;
                    const uint32_t st = gp % L::kStages;
                    if (!(ok = sync.wait(bar(kBarKvFull + st), (gp / L::kStages) & 1))) break;
                    tc_fence_after();
                    const uint32_t s_tmem = tmem + kTmemS + 64 * (gp & 1);
                    const uint32_t k_base = s_kv + st * L::kStageBytes;
#pragma unroll
                    for (int ks = 0; ks < L::kKSlices; ++ks) {
                        uint64_t qd, kd;
                        if (ks < L::kBoxes * 4) {
                            const int box = ks >> 2, sub = ks & 3;
                            qd = smem_desc(s_q + box * 16384 + sub * 32, 16, 1024, kLayoutSW128);
                            kd = smem_desc(k_base + box * 8192 + sub * 32, 16, 1024, kLayoutSW128);
                        } else {
                            const int sub = ks - L::kBoxes * 4;
                            qd = smem_desc(s_q + L::kBoxes * 16384 + sub * 32, 16, 512, kLayoutSW64);
                            kd = smem_desc(k_base + L::kBoxes * 8192 + sub * 32, 16, 512, kLayoutSW64);
                        }
                        mma_ss(s_tmem, qd, kd, idesc_qk, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(kBarSFull + (gp & 1)));
                    if (j == n - 1) mma_commit(bar(kBarQFree));
                    if (j > 0) ok = issue_pv(gp - 1, j == 1);
                }
                if (ok) ok = issue_pv(g + n - 1, n == 1);
                if (ok) mma_commit(bar(kBarOFull));
                g += n;
                ++k;
            }
            // All issued MMAs complete before tensor memory is released.
            mma_commit(bar(kBarDrain));
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar(kBarDrain), 0) && global_timer_ns() - t0 < 100000000ull) {
            }
        }
    } else {
        // ======================= softmax / correction / epilogue =======================
        const int r = threadIdx.x;  // TMEM lane == query row within the row group
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t x_row = s_x + r * 256;
        const uint32_t x_row_peer = map_to_cta(x_row, peer);
        const uint32_t x_full_peer = map_to_cta(bar(kBarXFull + warp), peer);
        const uint32_t x_free_peer = map_to_cta(bar(kBarXFree + warp), peer);
        // Waits are made warp-uniform: the tcgen05 loads / stores below are warp-collective.
        auto wwait = [&](uint32_t b_, uint32_t par) { return __all_sync(0xffffffffu, sync.wait(b_, par)); };
        uint32_t g = 0, k = 0;
        int vb, lo, hi;
        bool ok = true;
        while (ok && chunks.next(vb, lo, hi)) {
            const int b = vb / p.groups, rg = vb % p.groups;
            const int Lb = p.seqlens[b];
            const int row = rg * kRowsPerGroup + r;
            const bool row_valid = row < p.rows;
            const int s_tok = row / p.h_q;
            int n_vis = Lb;
            if (p.causal) n_vis = min(max(Lb - p.s_q + 1 + s_tok, 0), Lb);
            const int nsplit = p.num_splits[vb + 1] - p.num_splits[vb];
            const int split_idx = (vb == begin_vb) ? begin_split : 0;
            const int n = hi - lo;
            const int last_page = pages_of(Lb) - 1;
            float m_ref = -INFINITY, l_sum = 0.f;

            for (int j = 0; j < n; ++j) {
                const uint32_t gp = g + j;
                const uint32_t sb = gp & 1;
                const uint32_t s_tmem = tmem + kTmemS + 64 * sb + lane_base;
                if (!(ok = wwait(bar(kBarSFull + sb), (gp >> 1) & 1))) break;
                tc_fence_after();
                float s[64];
                {
                    uint32_t a[32], c[32];
                    tmem_ld32(s_tmem, a);
                    tmem_ld32(s_tmem + 32, c);
                    tmem_wait_ld();
                    reg_fence(a);
                    reg_fence(c);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        s[i] = __uint_as_float(a[i]);
                        s[32 + i] = __uint_as_float(c[i]);
                    }
                }
                // ---- exchange partial logits with the peer CTA
                if (!(ok = wwait(bar(kBarXFree + warp), (gp & 1) ^ 1))) break;
                if (lane == 0) mbar_arrive_expect_tx(bar(kBarXFull + warp), 32 * 256);
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) {
                    const uint32_t off = ((c4 ^ (r & 15)) << 4);
                    st_async_v4(x_row_peer + off, s[4 * c4], s[4 * c4 + 1], s[4 * c4 + 2], s[4 * c4 + 3],
                                x_full_peer);
                }
                if (!(ok = wwait(bar(kBarXFull + warp), gp & 1))) break;
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) {
                    const uint32_t off = ((c4 ^ (r & 15)) << 4);
                    float4 t;
                    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                 : "=f"(t.x), "=f"(t.y), "=f"(t.z), "=f"(t.w)
                                 : "r"(x_row + off));
                    s[4 * c4] += t.x;
                    s[4 * c4 + 1] += t.y;
                    s[4 * c4 + 2] += t.z;
                    s[4 * c4 + 3] += t.w;
                }
                mbar_arrive_remote(x_free_peer);

                // ---- mask, scale, running maximum
                const int tok0 = (lo + j) * kPage;
                const int lim = n_vis - tok0;  // columns >= lim are not visible
                float mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    s[c] = (c < lim) ? s[c] * p.scale_log2 : -INFINITY;
                    mx = fmaxf(mx, s[c]);
                }
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
                float rs = 0.f;
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float p0 = fast_exp2(s[2 * c] - ref);
                    const float p1 = fast_exp2(s[2 * c + 1] - ref);
                    rs += p0 + p1;
                    pk[c] = pack2(p0, p1, kFp16);
                }
                l_sum = l_sum * alpha + rs;

                // ---- previous PV done: P buffer and O are ours
                if (j > 0 && !(ok = wwait(bar(kBarPvDone), (gp - 1) & 1))) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, rescale)) {
                    const float a = rescale ? alpha : 1.f;
#pragma unroll 1
                    for (int cb = 0; cb < kDvHalf / 32; ++cb) {
                        uint32_t v[32];
                        tmem_ld32(tmem + kTmemO + lane_base + 32 * cb, v);
                        tmem_wait_ld();
                        reg_fence(v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * a);
                        tmem_st32(tmem + kTmemO + lane_base + 32 * cb, v);
                    }
                }
                // ---- the sequence's last, partly filled page: zero V rows past the end so
                //      that whatever the cache holds there cannot reach O through 0 * x.
                if (lo + j == last_page && (Lb % kPage) != 0) {
                    const int tail = Lb % kPage;
                    const uint32_t st = gp % L::kStages;
                    uint8_t* stage = smem + L::kOffKV + st * L::kStageBytes;
                    const int per_box = (kPage - tail) * 128 / 16;
                    for (int i = r; i < per_box * L::kBoxes; i += 128) {
                        const int box = i / per_box, w16 = i % per_box;
                        *reinterpret_cast<uint4*>(stage + box * 8192 + tail * 128 + w16 * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                }
                tmem_st32(s_tmem, pk);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarPFull));
            }
            if (!ok) break;

            // ---- epilogue
            const bool empty = (n <= 0);
            const float inv_l = (l_sum > 0.f) ? 1.f / l_sum : 0.f;
            const float lse_v = (l_sum > 0.f) ? (m_ref + log2f(l_sum)) * 0.69314718055994531f : -INFINITY;
            if (!empty) {
                if (!(ok = wwait(bar(kBarOFull), k & 1))) break;
                tc_fence_after();
            }
            if (nsplit == 1) {
                typedef uint4 vec_t;
                vec_t* dst = reinterpret_cast<vec_t*>(static_cast<uint8_t*>(p.o) +
                                                      ((static_cast<size_t>(b) * p.rows + row) * kDv + col0) * 2);
#pragma unroll 1
                for (int cb = 0; cb < kDvHalf / 32; ++cb) {
                    uint32_t v[32];
                    if (!empty) {
                        tmem_ld32(tmem + kTmemO + lane_base + 32 * cb, v);
                        tmem_wait_ld();
                        reg_fence(v);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = 0;
                    }
                    uint32_t h[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        h[i] = pack2(__uint_as_float(v[2 * i]) * inv_l, __uint_as_float(v[2 * i + 1]) * inv_l, kFp16);
                    if (row_valid) {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[cb * 4 + i] = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
                    }
                }
                if (cta == 0 && row_valid) p.lse[static_cast<size_t>(b) * p.rows + row] = lse_v;
            } else {
                const size_t slot = static_cast<size_t>(p.num_splits[vb]) + split_idx;
                float4* dst = reinterpret_cast<float4*>(p.o_accum + (slot * kRowsPerGroup + r) * kDv + col0);
#pragma unroll 1
                for (int cb = 0; cb < kDvHalf / 32; ++cb) {
                    uint32_t v[32];
                    if (!empty) {
                        tmem_ld32(tmem + kTmemO + lane_base + 32 * cb, v);
                        tmem_wait_ld();
                        reg_fence(v);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = 0;
                    }
                    if (row_valid) {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            dst[cb * 8 + i] = make_float4(__uint_as_float(v[4 * i]) * inv_l,
                                                          __uint_as_float(v[4 * i + 1]) * inv_l,
                                                          __uint_as_float(v[4 * i + 2]) * inv_l,
                                                          __uint_as_float(v[4 * i + 3]) * inv_l);
                    }
                }
                if (cta == 0) p.lse_accum[slot * kRowsPerGroup + r] = lse_v;
            }
            if (!empty) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarOFree));
                ++k;
            }
            g += (n > 0 ? n : 0);
        }
    }

    // ---------------- teardown
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no remote access to this CTA's shared memory after this point
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ combine kernel
// Merges the split partial results of every virtual batch with more than one
// split: lse = log sum_k exp(lse_k), o = sum_k exp(lse_k - lse) o_k.  One warp
// per query row; lane i owns 16 of the 512 output columns.
template <bool kFp16>
__global__ void __launch_bounds__(256) mla_combine_kernel(DecodeParams p)
{
    const int vb = blockIdx.x;
    const int nsplit = p.num_splits[vb + 1] - p.num_splits[vb];
    if (nsplit <= 1) return;
    const int b = vb / p.groups, rg = vb % p.groups;
    const int slot0 = p.num_splits[vb];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rows_here = min(kRowsPerGroup, p.rows - rg * kRowsPerGroup);
    for (int r = blockIdx.y * 8 + warp; r < rows_here; r += gridDim.y * 8) {
        float mx = -INFINITY;
        for (int k = lane; k < nsplit; k += 32) mx = fmaxf(mx, p.lse_accum[(size_t)(slot0 + k) * kRowsPerGroup + r]);
#pragma unroll
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.f;
        if (mx != -INFINITY)
            for (int k = lane; k < nsplit; k += 32)
                sum += expf(p.lse_accum[(size_t)(slot0 + k) * kRowsPerGroup + r] - mx);
#pragma unroll
        for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float lse = (mx == -INFINITY) ? -INFINITY : mx + logf(sum);
        float acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = 0.f;
        if (mx != -INFINITY) {
            for (int k = 0; k < nsplit; ++k) {
                const float w = expf(p.lse_accum[(size_t)(slot0 + k) * kRowsPerGroup + r] - lse);
                if (w == 0.f) continue;
                const float4* src =
                    reinterpret_cast<const float4*>(p.o_accum + ((size_t)(slot0 + k) * kRowsPerGroup + r) * kDv);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 v = src[lane + 32 * i];
                    acc[4 * i] += w * v.x;
                    acc[4 * i + 1] += w * v.y;
                    acc[4 * i + 2] += w * v.z;
                    acc[4 * i + 3] += w * v.w;
                }
            }
        }
        const int row = rg * kRowsPerGroup + r;
        uint2* dst = reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.o) + ((size_t)b * p.rows + row) * kDv * 2);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            dst[lane + 32 * i] = make_uint2(pack2(acc[4 * i], acc[4 * i + 1], kFp16), pack2(acc[4 * i + 2], acc[4 * i + 3], kFp16));
        if (lane == 0) p.lse[(size_t)b * p.rows + row] = lse;
    }
}

// ------------------------------------------------------------------ metadata kernel
__global__ void mla_metadata_kernel(const int32_t* seqlens, int batch, int groups, int num_parts, int32_t* md,
                                    int32_t* num_splits, int32_t* scratch_unused)
{
    extern __shared__ int32_t s_len[];
    for (int i = threadIdx.x; i < batch; i += blockDim.x) s_len[i] = seqlens[i];
    __syncthreads();
    if (threadIdx.x == 0) schedule(s_len, batch, groups, num_parts, md, num_splits);
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

static size_t workspace_slots(int batch, int groups, int num_parts)
{
    return static_cast<size_t>(batch) * groups + static_cast<size_t>(num_parts);
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

template <bool kRope, bool kFp16>
static cudaError_t launch_splitkv(int grid, cudaStream_t stream, const CUtensorMap& q128, const CUtensorMap& q64,
                                  const CUtensorMap& kv128, const CUtensorMap& kv64, const DecodeParams& prm)
{
    auto kern = mla_splitkv_kernel<kRope, kFp16>;
    const int smem = Layout<kRope>::kSmemBytes;
    static int configured_device = -1;  // attribute is per device; set it once per device in use
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_device != dev) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    kern<<<grid, kThreads, smem, stream>>>(q128, q64, kv128, kv64, prm);
    return cudaGetLastError();
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
                                 int num_parts, int32_t* tile_md, int32_t* num_splits)
{
    if (batch < 0 || heads_per_kv <= 0 || h_kv <= 0 || num_parts <= 0 || !tile_md || !num_splits ||
        (batch > 0 && !cache_seqlens))
        return MLA_ERR_INVALID_ARG;
    if (h_kv != 1) return MLA_ERR_UNSUPPORTED;
    for (int b = 0; b < batch; ++b)
        if (cache_seqlens[b] < 0) return MLA_ERR_INVALID_ARG;
    schedule(cache_seqlens, batch, row_groups(heads_per_kv), num_parts, tile_md, num_splits);
    return MLA_OK;
}

mla_status mla_get_metadata(const int32_t* cache_seqlens, int batch, int heads_per_kv, int h_kv, int num_parts,
                            int32_t* tile_md, int32_t* num_splits, void* stream)
{
    if (batch < 0 || heads_per_kv <= 0 || h_kv <= 0 || num_parts <= 0 || !tile_md || !num_splits ||
        (batch > 0 && !cache_seqlens))
        return MLA_ERR_INVALID_ARG;
    if (h_kv != 1) return MLA_ERR_UNSUPPORTED;
    if (batch > 12000) return MLA_ERR_UNSUPPORTED;  // sequence lengths are staged in shared memory
    mla_metadata_kernel<<<1, 256, static_cast<size_t>(batch) * sizeof(int32_t) + 16,
                          static_cast<cudaStream_t>(stream)>>>(cache_seqlens, batch, row_groups(heads_per_kv),
                                                               num_parts, tile_md, num_splits, nullptr);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

size_t mla_decode_workspace_bytes(int batch, int s_q, int h_q, int h_kv, int num_parts)
{
    if (batch < 0 || s_q <= 0 || h_q <= 0 || h_kv <= 0 || num_parts <= 0 || h_q % h_kv) return 0;
    const int groups = row_groups(s_q * h_q / h_kv);
    const size_t slots = workspace_slots(batch, groups, num_parts);
    size_t bytes = kWorkspaceHeader;
    bytes += align_up(slots * kRowsPerGroup * sizeof(float), 256);
    bytes += slots * kRowsPerGroup * kDv * sizeof(float);
    return bytes;
}

// Validates the arguments and fills the kernel parameters and tensor maps.
static mla_status prepare_decode(const void* q, int batch, int s_q, int h_q, int d_qk, const void* kvcache,
                                 int num_blocks, int page_size, int h_kv, const int32_t* block_table,
                                 int max_blocks_per_seq, const int32_t* cache_seqlens, int dv, int dtype,
                                 const int32_t* tile_md, int num_parts, const int32_t* num_splits, int causal,
                                 float softmax_scale, void* o, float* lse, void* workspace, size_t workspace_bytes,
                                 DecodeParams& prm, CUtensorMap* maps)
{
    if (batch < 0 || s_q <= 0 || h_q <= 0 || h_kv <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 ||
        num_parts <= 0 || (causal != 0 && causal != 1))
        return MLA_ERR_INVALID_ARG;
    if (dtype != MLA_BF16 && dtype != MLA_FP16) return MLA_ERR_INVALID_ARG;
    if (page_size != kPage || h_kv != 1 || (d_qk != 576 && d_qk != 512) || dv != kDv) return MLA_ERR_UNSUPPORTED;
    if (batch > 0 && (!q || !kvcache || !block_table || !cache_seqlens || !tile_md || !num_splits || !o || !lse ||
                      !workspace))
        return MLA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(kvcache) & 15) ||
        (reinterpret_cast<uintptr_t>(o) & 15) || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return MLA_ERR_INVALID_ARG;
    const int rows = s_q * h_q;
    const int groups = row_groups(rows);
    const size_t need = mla_decode_workspace_bytes(batch, s_q, h_q, h_kv, num_parts);
    if (batch > 0 && workspace_bytes < need) return MLA_ERR_WORKSPACE;
    if (static_cast<long long>(num_blocks) * kPage >= (1ll << 31)) return MLA_ERR_UNSUPPORTED;
    if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt(static_cast<float>(d_qk));
    prm = DecodeParams{};
    prm.block_table = block_table;
    prm.seqlens = cache_seqlens;
    prm.md = tile_md;
    prm.num_splits = num_splits;
    prm.o = o;
    prm.lse = lse;
    prm.batch = batch;
    prm.s_q = s_q;
    prm.h_q = h_q;
    prm.rows = rows;
    prm.groups = groups;
    prm.max_blocks = max_blocks_per_seq;
    prm.num_blocks = num_blocks;
    prm.causal = causal;
    prm.box_rows = rows < kRowsPerGroup ? rows : kRowsPerGroup;
    prm.scale_log2 = softmax_scale * 1.4426950408889634f;
    prm.dtype = dtype;
    prm.d_qk = d_qk;
    prm.num_parts = num_parts;
    if (batch == 0) return MLA_OK;
    const size_t slots = workspace_slots(batch, groups, num_parts);
    prm.status = static_cast<int*>(workspace);
    prm.lse_accum = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWorkspaceHeader);
    prm.o_accum = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWorkspaceHeader +
                                           align_up(slots * kRowsPerGroup * sizeof(float), 256));
    if (!maps) return MLA_OK;

    const CUtensorMapDataType dt =
        dtype == MLA_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const uint64_t row_bytes = static_cast<uint64_t>(d_qk) * 2;
    const uint64_t kv_rows = static_cast<uint64_t>(num_blocks) * kPage;
    bool ok = encode_3d(&maps[0], q, dt, d_qk, rows, batch, row_bytes, row_bytes * rows, 64, prm.box_rows,
                        CU_TENSOR_MAP_SWIZZLE_128B) &&
              encode_2d(&maps[2], kvcache, dt, d_qk, kv_rows, row_bytes, 64, kPage, CU_TENSOR_MAP_SWIZZLE_128B);
    if (ok && d_qk == 576)
        ok = encode_3d(&maps[1], q, dt, d_qk, rows, batch, row_bytes, row_bytes * rows, 32, prm.box_rows,
                       CU_TENSOR_MAP_SWIZZLE_64B) &&
             encode_2d(&maps[3], kvcache, dt, d_qk, kv_rows, row_bytes, 32, kPage, CU_TENSOR_MAP_SWIZZLE_64B);
    else {
        maps[1] = maps[0];
        maps[3] = maps[2];
    }
    return ok ? MLA_OK : MLA_ERR_CUDA;
}

static mla_status launch_splitkv_stage(const DecodeParams& prm, const CUtensorMap* maps, cudaStream_t st)
{
    const int grid = 2 * prm.num_parts;
    cudaError_t e;
    if (prm.d_qk == 576)
        e = prm.dtype == MLA_FP16 ? launch_splitkv<true, true>(grid, st, maps[0], maps[1], maps[2], maps[3], prm)
                                  : launch_splitkv<true, false>(grid, st, maps[0], maps[1], maps[2], maps[3], prm);
    else
        e = prm.dtype == MLA_FP16 ? launch_splitkv<false, true>(grid, st, maps[0], maps[1], maps[2], maps[3], prm)
                                  : launch_splitkv<false, false>(grid, st, maps[0], maps[1], maps[2], maps[3], prm);
    return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

static mla_status launch_combine_stage(const DecodeParams& prm, cudaStream_t st)
{
    dim3 cgrid(prm.batch * prm.groups, 4);
    if (prm.dtype == MLA_FP16)
        mla_combine_kernel<true><<<cgrid, 256, 0, st>>>(prm);
    else
        mla_combine_kernel<false><<<cgrid, 256, 0, st>>>(prm);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

#define MLA_DECODE_ARGS                                                                                          \
    q, batch, s_q, h_q, d_qk, kvcache, num_blocks, page_size, h_kv, block_table, max_blocks_per_seq,            \
        cache_seqlens, dv, dtype, tile_md, num_parts, num_splits, causal, softmax_scale, o, lse, workspace,      \
        workspace_bytes

mla_status mla_decode_with_kvcache(const void* q, int batch, int s_q, int h_q, int d_qk, const void* kvcache,
                                   int num_blocks, int page_size, int h_kv, const int32_t* block_table,
                                   int max_blocks_per_seq, const int32_t* cache_seqlens, int dv, int dtype,
                                   const int32_t* tile_md, int num_parts, const int32_t* num_splits, int causal,
                                   float softmax_scale, void* o, float* lse, void* workspace,
                                   size_t workspace_bytes, void* stream)
{
    DecodeParams prm;
    CUtensorMap maps[4];
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
                              float softmax_scale, void* o, float* lse, void* workspace, size_t workspace_bytes,
                              void* stream)
{
    DecodeParams prm;
    CUtensorMap maps[4];
    mla_status s = prepare_decode(MLA_DECODE_ARGS, prm, maps);
    if (s != MLA_OK || batch == 0) return s;
    return launch_splitkv_stage(prm, maps, static_cast<cudaStream_t>(stream));
}

mla_status mla_decode_combine(int batch, int s_q, int h_q, int h_kv, int dv, int dtype, const int32_t* num_splits,
                              int num_parts, void* o, float* lse, void* workspace, size_t workspace_bytes,
                              void* stream)
{
    if (batch < 0 || s_q <= 0 || h_q <= 0 || h_kv <= 0 || num_parts <= 0) return MLA_ERR_INVALID_ARG;
    if (dtype != MLA_BF16 && dtype != MLA_FP16) return MLA_ERR_INVALID_ARG;
    if (h_kv != 1 || dv != kDv) return MLA_ERR_UNSUPPORTED;
    if (batch == 0) return MLA_OK;
    if (!num_splits || !o || !lse || !workspace) return MLA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return MLA_ERR_INVALID_ARG;
    if (workspace_bytes < mla_decode_workspace_bytes(batch, s_q, h_q, h_kv, num_parts)) return MLA_ERR_WORKSPACE;
    const int rows = s_q * h_q;
    const int groups = row_groups(rows);
    const size_t slots = workspace_slots(batch, groups, num_parts);
    DecodeParams prm{};
    prm.num_splits = num_splits;
    prm.o = o;
    prm.lse = lse;
    prm.rows = rows;
    prm.groups = groups;
    prm.batch = batch;
    prm.dtype = dtype;
    prm.lse_accum = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWorkspaceHeader);
    prm.o_accum = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWorkspaceHeader +
                                           align_up(slots * kRowsPerGroup * sizeof(float), 256));
    return launch_combine_stage(prm, static_cast<cudaStream_t>(stream));
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
    if (clear && cudaMemsetAsync(workspace, 0, sizeof(int), st) != cudaSuccess) return MLA_ERR_CUDA;
    return MLA_OK;
}

}  // extern "C"
