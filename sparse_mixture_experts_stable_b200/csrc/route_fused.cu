// Router scores, softmax, stable top-k and gates in one kernel (bf16
// activations and router weight, fp32 accumulation in tensor memory).
//
// The router page's problem is one pass over the activations: s = x . W_r for
// every token, then a softmax and a top-k per token.  Writing s to memory and
// reading it back costs more than a quarter of the pass, so here the scores
// never leave the SM: each 128-token tile is multiplied on tcgen05 into a
// 128 x E fp32 accumulator in TMEM, and sixteen epilogue warps take it apart
// in registers.
//
// Work split: CTAs run in pairs (a two-CTA cluster on two SMs) that share one
// tcgen05 MMA of 256 tokens x E experts: each CTA stages its own 128 token
// rows and half of the router weight's rows, and receives its tokens' 128 x E
// scores in its own tensor memory.  Sharing the weight halves the bytes each
// SM pulls from L2 per k-block (16 KB of weight beside 16 KB of activations,
// against 32 KB + 16 KB for a CTA alone), and one thread issues the MMAs of
// two SMs.  Every pair owns one contiguous run of tokens balanced to 32 rows
// across the grid; a run is processed in pair tiles of up to 256 tokens, and
// only the 32-row TMA boxes that hold the run's own rows are loaded.
//
// Warp roles (608 threads per CTA):
//   warp 0      TMA producer of the CTA's token rows
//   warp 1      TMA producer of the CTA's half of the router weight (re-read
//               from L2 for every tile)
//   warp 2      TMEM owner (both CTAs) and MMA issuer (one lane of the even
//               CTA): two E-column accumulators, so a tile's epilogue overlaps
//               the next tile's main loop
// Both CTAs' producers feed one ring of five 32 KB stages: k-block g's four
// loads land on the even CTA's full[g % 5], whose two producers arm it with
// the bytes of both CTAs (the odd CTA's producers only issue their loads), and
// the MMA commit releases empty[g % 5] in both CTAs.  One wait and one commit per k-block keep the
// issuing thread's work between two k-blocks short, and the next k-block's
// barrier is tested while the current one's MMAs are being accepted, since
// the tensor core takes new MMAs only as it finishes old ones: a late look at
// the barrier leaves it idle.
//   warps 3-18  epilogue: warp w reads TMEM lanes 32*(w%4).. (its 32 tokens)
//               and one quarter of the E columns, 32 columns per TMEM load.
//
// The epilogue finds the top-8 without ranking every score against a list:
//   pass 1  each 32-score chunk is sorted in groups of eight by a 19-comparator
//           network and the groups are merged by bitonic half-cleaners, so the
//           chunk's eight largest VALUES cost about eight min/max operations
//           per score; the quarter keeps its eight largest values and an
//           online softmax sum (the chunk maximum is the largest group head).
//   exchange  the four quarters of a token publish their value lists and sums
//           through shared memory; every thread merges them in a fixed order,
//           which gives the token's exact eighth-largest score tau, its maximum
//           and its softmax denominator.
//   pass 2  re-reads the accumulator for the probabilities (summed over the
//           warp's 32 tokens per expert) and collects the candidates: a score
//           above tau (at most seven per token) goes to a value slot, a score
//           equal to tau only sets a bit, since its value is known.
//   select  each thread inserts its candidates into a list ordered by (score
//           descending, expert index ascending), the slots first and then the
//           tied experts in ascending order; the four lists are merged in two
//           rounds and the first quarter writes selected, gates and counts.
// Every score below tau is outside the top-8 and every score above it inside,
// so the candidates hold the whole answer and the ordered insertion makes the
// tie-break exact.
// Per-expert probability sums are reduced over the 32 tokens of a warp with a
// fixed butterfly, kept in registers across tiles and added in a fixed order
// at the end, so prob_sum stays bitwise reproducible for a given grid.
//
// The exponentials are ex2.approx of (score - max) * log2(e) (a fused
// multiply-add); its documented relative error is a few ulp, far below the
// tolerances of the probability sums and the gates.
//
// Every mbarrier wait is bounded; after a timeout the producers and the MMA
// issuer stop, and the epilogue runs its remaining tiles without writing
// anything, so the named barriers between its warps and the closing cluster
// barrier always complete.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "route_fused.cuh"
#include "tc_gemm.cuh"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace tc;

constexpr int kRM = 128;       // tokens per tile (UMMA M)
constexpr int kRBK = 64;       // K per stage (64 bf16 = one 128-byte swizzle row)
constexpr int kRStages = 5;
constexpr int kRBox = 32;      // token rows per TMA box
constexpr int kREpiWarps = 16;
constexpr int kRThreads = (3 + kREpiWarps) * 32;
constexpr int kRABytes = kRM * kRBK * 2;  // 16 KB
constexpr int kRTopK = 8;
constexpr int kRE = 256;                  // experts (the fused path's only width)
constexpr int kRCQ = kRE / 4;             // columns per epilogue quarter
constexpr int kRBBytes = (kRE / 2) * kRBK * 2;  // this CTA's half of the weight: 16 KB
constexpr int kRStageBytes = kRABytes + kRBBytes;

// Shared memory of one lane-quarter group (the 4 epilogue warps that read the
// same 32 TMEM lanes): an 8 KB area that holds first the exchange of the
// quarters' (top-8 values, softmax sum, finiteness) and then the value slots
// of the candidates above tau, and a 4 KB area for the two lists in transit
// of the final merge.
constexpr int kExWords = kRTopK + 2;         // per (quarter, token): 8 values, sum, finite flag
constexpr int kSlots = kRTopK;               // 7 candidates at most (one spare)
constexpr int kGroupUnion = kSlots * 128 * 8;  // 8 KB
constexpr int kGroupMerge = 2 * kRTopK * 32 * 8;  // 4 KB
static_assert(4 * kExWords * 32 * 4 <= kGroupUnion, "exchange must fit the union area");

// dynamic shared memory layout (offsets from a 1024-byte aligned base)
constexpr size_t kOffStages = 0;  // stage s: A at s * 32 KB, the weight half 16 KB after it
constexpr size_t kOffBars = kOffStages + (size_t)kRStages * kRStageBytes;
constexpr size_t kOffMisc = kOffBars + 256;
constexpr size_t kOffBias = kOffMisc + 64;
constexpr size_t kOffCounts = kOffBias + kRE * 4;
constexpr size_t kOffUnion = kOffCounts + kRE * 4;
constexpr size_t kOffMerge = kOffUnion + 4 * (size_t)kGroupUnion;
constexpr size_t kSmemBytes = kOffMerge + 4 * (size_t)kGroupMerge;
static_assert(kSmemBytes <= 232448, "the router kernel must fit one SM's shared memory");
static_assert(4 * kRE * 4 <= 4 * kGroupUnion, "final per-group sums reuse the union area");

struct RFParams {
    int64_t T;
    int64_t units;  // ceil(T / 32)
    int k;
    int k_blocks;
    const float* bias;
    float* logits_out;
    int64_t* selected;
    void* gates;
    int gates_bf16;
    float* gates_f32;
    int32_t* part_counts;
    float* part_psum;
    int32_t* status;
};

__device__ __forceinline__ void named_bar(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Insert (v, idx) into a list sorted by (score descending, index ascending).
// Every candidate has a higher index than the entries of equal score already in
// the list (a quarter's experts arrive in ascending order; a merged list's
// entries all lie above the receiving list's and arrive in its own order), so
// the new entry goes before the first strictly smaller score, and the entries
// from there on shift down by one place unconditionally: ties keep the lower
// expert index first.  The eight comparisons are independent of each other.
__device__ __forceinline__ void topk_insert(float (&tv)[kRTopK], int (&ti)[kRTopK], float v, int idx) {
    bool p[kRTopK];
#pragma unroll
    for (int j = 0; j < kRTopK; ++j) p[j] = v > tv[j];  // monotone: false ... false true ... true
#pragma unroll
    for (int j = kRTopK - 1; j >= 1; --j) {
        tv[j] = p[j] ? (p[j - 1] ? tv[j - 1] : v) : tv[j];
        ti[j] = p[j] ? (p[j - 1] ? ti[j - 1] : idx) : ti[j];
    }
    tv[0] = p[0] ? v : tv[0];
    ti[0] = p[0] ? idx : ti[0];
}

// compare-exchange for a descending order (values only)
__device__ __forceinline__ void cx(float& a, float& b) {
    const float hi = fmaxf(a, b);
    b = fminf(a, b);
    a = hi;
}

// sorts a[0..7] descending: the 19-comparator, depth-6 network of Knuth's
// Sorting and Searching (section 5.3.4), checked on all 0-1 inputs
__device__ __forceinline__ void sort8_desc(float* a) {
    cx(a[0], a[2]); cx(a[1], a[3]); cx(a[4], a[6]); cx(a[5], a[7]);
    cx(a[0], a[4]); cx(a[1], a[5]); cx(a[2], a[6]); cx(a[3], a[7]);
    cx(a[0], a[1]); cx(a[2], a[3]); cx(a[4], a[5]); cx(a[6], a[7]);
    cx(a[2], a[4]); cx(a[3], a[5]);
    cx(a[1], a[4]); cx(a[3], a[6]);
    cx(a[1], a[2]); cx(a[3], a[4]); cx(a[5], a[6]);
}

// a <- the eight largest of a and b (both sorted descending), sorted
// descending: max(a_i, b_(7-i)) is bitonic and holds the eight largest, and
// three half-cleaner stages sort it
__device__ __forceinline__ void merge8_desc(float* a, const float* b) {
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = fmaxf(a[i], b[7 - i]);
#pragma unroll
    for (int d = 4; d >= 1; d >>= 1)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (!(i & d)) cx(a[i], a[i + d]);
}

// Lane l returns the sum over the warp's lanes of a[l] (a is overwritten).
__device__ __forceinline__ float transpose_sum32(float* a, int lane) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int j = 0; j < o; ++j) {
            const float send = up ? a[j] : a[j + o];
            const float keep = up ? a[j + o] : a[j];
            a[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return a[0];
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kRThreads, 1)
    route_fused_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                       const RFParams p) {
    constexpr int E = kRE;
    constexpr int CQ = kRCQ;
    constexpr float kLog2e = 1.4426950408889634f;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if ((smem_u32(smem_raw) & 1023u) != 0) {  // the layout needs a 1024-byte aligned base (swizzled stages)
        if (threadIdx.x == 0) set_status(p.status, MOE_ERR_CUDA);
        return;
    }
    uint8_t* stages = smem_raw + kOffStages;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + kOffBars);
    uint64_t* full = bars;                 // even CTA: k-block g's four loads have landed
    uint64_t* empty = bars + kRStages;     // both CTAs: k-block g's MMAs are done
    uint64_t* tfull = bars + 2 * kRStages; // both CTAs: the accumulator holds a finished tile
    uint64_t* tempty = tfull + 2;          // even CTA: both CTAs' epilogues released the accumulator
    uint32_t* s_tmem_p = reinterpret_cast<uint32_t*>(smem_raw + kOffMisc);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem_raw + kOffMisc + 4);
    float* s_bias = reinterpret_cast<float*>(smem_raw + kOffBias);
    int* s_counts = reinterpret_cast<int*>(smem_raw + kOffCounts);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();  // 0: issues the MMAs; 1: its partner
    const bool leader = rank == 0;

    // the pair's run of tokens, balanced in 32-row units; pair tile i holds rows
    // row_begin + 256 i .. + 256, this CTA the half starting at 128 * rank
    const int64_t pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const int64_t u0 = pair * p.units / n_pairs;
    const int64_t u1 = (pair + 1) * p.units / n_pairs;
    const int64_t row_begin = u0 * kRBox;
    const int64_t row_end = u1 * kRBox < p.T ? u1 * kRBox : p.T;
    const int n_tiles = row_end > row_begin ? (int)((row_end - row_begin + 2 * kRM - 1) / (2 * kRM)) : 0;
    // the even CTA's barriers, as shared::cluster addresses
    const uint32_t full_l = mapa_shared(smem_u32(full), 0);
    const uint32_t tempty_l = mapa_shared(smem_u32(tempty), 0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRStages; ++s) {
            mbar_init(&full[s], 2);  // the even CTA's A and weight producers
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 2 * kREpiWarps);  // one arrival per epilogue warp of either CTA
        }
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW)) : "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem_p)),
                     "r"(2 * E)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        s_bias[e] = p.bias ? p.bias[e] : 0.f;
        s_counts[e] = 0;
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers are initialised before either signals the other's
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem_p;

    if (warp == 0) {
        // ------------------------- token-row producer -------------------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int i = 0; i < n_tiles && !*s_abort; ++i) {
                const int64_t rp = row_begin + (int64_t)i * 2 * kRM;  // the pair tile's first row
                auto boxes = [&](int64_t r) {  // 32-row boxes of the half starting at row r
                    const int64_t n = row_end - r < kRM ? (row_end > r ? row_end - r : 0) : kRM;
                    return (int)((n + kRBox - 1) / kRBox);
                };
                const int64_t r0 = rp + (int64_t)rank * kRM;
                const int nbox = boxes(r0);
                const uint32_t pair_bytes = (uint32_t)((boxes(rp) + boxes(rp + kRM)) * kRBox * kRBK * 2);
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.status)) {  // k-block g - 5 is done
                        *s_abort = 1;
                        break;
                    }
                    const uint32_t fb = full_l + 8u * (uint32_t)stage;
                    if (leader) mbar_expect_tx(&full[stage], pair_bytes);
                    uint8_t* dst = stages + stage * kRStageBytes;
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d_pair(dst + b * (kRBox * kRBK * 2), &tmX, kb * kRBK, (int32_t)(r0 + b * kRBox), fb);
                    if (++stage == kRStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------ router-weight producer -----------------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int i = 0; i < n_tiles && !*s_abort; ++i) {
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, p.status)) {
                        *s_abort = 1;
                        break;
                    }
                    const uint32_t fb = full_l + 8u * (uint32_t)stage;
                    if (leader) mbar_expect_tx(&full[stage], 2u * (uint32_t)kRBBytes);
                    tma_load_2d_pair(stages + stage * kRStageBytes + kRABytes, &tmW, kb * kRBK,
                                     (int32_t)(rank * (kRE / 2)), fb);
                    if (++stage == kRStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 2) {
        // ------------------------------ MMA issuer -----------------------------
        if (lane == 0 && leader) {
            const uint32_t idesc = make_idesc(2 * kRM, E);
            int sa = 0;
            uint32_t pa = 0;
            const uint32_t full0 = smem_u32(full);
            bool ready = mbar_test(full0, 0u);
            for (int i = 0; i < n_tiles && !*s_abort; ++i) {
                const uint32_t acc = (uint32_t)i & 1u;
                if (!mbar_wait_cluster(&tempty[acc], (((uint32_t)i >> 1) & 1u) ^ 1u, p.status)) {
                    *s_abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * E;
                bool ok = true;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!ready && !mbar_wait(&full[sa], pa, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(smem_u32(stages + sa * kRStageBytes));
                    const uint64_t bd = sw128_desc(smem_u32(stages + sa * kRStageBytes + kRABytes));
                    const int sn = sa + 1 == kRStages ? 0 : sa + 1;
                    const uint32_t pn = sa + 1 == kRStages ? pa ^ 1u : pa;
                    tc_mma_pair(d_tmem, ad, bd, idesc, kb > 0 ? 1u : 0u);
                    tc_mma_pair(d_tmem, ad + 2, bd + 2, idesc, 1u);
                    ready = mbar_test(full0 + 8u * (uint32_t)sn, pn);  // the next k-block, early
                    tc_mma_pair(d_tmem, ad + 4, bd + 4, idesc, 1u);
                    tc_mma_pair(d_tmem, ad + 6, bd + 6, idesc, 1u);
                    tc_commit_pair(&empty[sa]);
                    sa = sn;
                    pa = pn;
                }
                if (!ok) {
                    *s_abort = 1;
                    break;
                }
                tc_commit_pair(&tfull[acc]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------- epilogue ------------------------------
        const int q = warp & 3;         // TMEM lane quarter this warp may read
        const int c = (warp - 3) >> 2;  // column quarter
        const int row = q * 32 + lane;
        const int tig = c * 32 + lane;  // thread within the lane-quarter group
        const int bar_id = 1 + q;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        float* s_ex = reinterpret_cast<float*>(smem_raw + kOffUnion + (size_t)q * kGroupUnion);  // [c][word][lane]
        uint8_t* s_slot = smem_raw + kOffUnion + (size_t)q * kGroupUnion;  // [slot][tig] x (value, index)
        float* s_mv = reinterpret_cast<float*>(smem_raw + kOffMerge + (size_t)q * kGroupMerge);  // [list][j][lane]
        int* s_mi = reinterpret_cast<int*>(smem_raw + kOffMerge + (size_t)q * kGroupMerge + kGroupMerge / 2);
        const uint32_t slot_base = smem_u32(s_slot) + (uint32_t)tig * 8u;
        const uint32_t slot_last = slot_base + (uint32_t)(kSlots - 1) * 1024u;
        float acc_ps[2] = {0.f, 0.f};

        for (int i = 0; i < n_tiles; ++i) {
            const uint32_t acc = (uint32_t)i & 1u;
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&tfull[acc], ((uint32_t)i >> 1) & 1u, p.status) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) *s_abort = 1;
            tc_fence_after();
            const int64_t r0 = row_begin + (int64_t)i * 2 * kRM + (int64_t)rank * kRM;
            const bool valid = r0 + row < row_end;
            const int64_t t = r0 + row;
            const bool write = valid && !*s_abort;
            const uint32_t tcol = tmem_base + acc * E + lane_off + (uint32_t)(c * CQ);

            // ---- pass 1: the quarter's eight largest values and its softmax sum ----
            float qt[kRTopK];
            float m_run = -INFINITY, ssum = 0.f, fin0 = 0.f, fin1 = 0.f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t r[32];
                tmem_ld32(tcol + 32 * h, r);
                tmem_ld_wait(r);
                float v[32];
                const float4* b4 = reinterpret_cast<const float4*>(s_bias + c * CQ + 32 * h);
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const float4 b = b4[j4];
                    v[4 * j4 + 0] = __uint_as_float(r[4 * j4 + 0]) + b.x;
                    v[4 * j4 + 1] = __uint_as_float(r[4 * j4 + 1]) + b.y;
                    v[4 * j4 + 2] = __uint_as_float(r[4 * j4 + 2]) + b.z;
                    v[4 * j4 + 3] = __uint_as_float(r[4 * j4 + 3]) + b.w;
                }
                // x * 0 is 0 for finite x and NaN for an infinity or a NaN
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    fin0 = fmaf(v[j], 0.f, fin0);
                    fin1 = fmaf(v[j + 1], 0.f, fin1);
                }
                if (p.logits_out && write) {
                    float4* dst = reinterpret_cast<float4*>(p.logits_out + t * E + c * CQ + 32 * h);
#pragma unroll
                    for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                }
#pragma unroll
                for (int g = 0; g < 4; ++g) sort8_desc(v + 8 * g);
                // online softmax: the chunk maximum is the largest group head
                const float cm = fmaxf(fmaxf(v[0], v[8]), fmaxf(v[16], v[24]));
                const float m_new = fmaxf(m_run, cm);
                const float mL = m_new == -INFINITY ? 0.f : m_new * kLog2e;
                float e0 = 0.f, e1 = 0.f;
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    e0 += ex2_approx(fmaf(v[j], kLog2e, -mL));
                    e1 += ex2_approx(fmaf(v[j + 1], kLog2e, -mL));
                }
                ssum = (m_run == m_new ? ssum : ssum * ex2_approx(fmaf(m_run, kLog2e, -mL))) + (e0 + e1);
                m_run = m_new;
                merge8_desc(v, v + 8);
                merge8_desc(v + 16, v + 24);
                merge8_desc(v, v + 16);
                if (h == 0) {
#pragma unroll
                    for (int j = 0; j < kRTopK; ++j) qt[j] = v[j];
                } else {
                    merge8_desc(qt, v);
                }
            }
            const bool q_finite = (fin0 + fin1) == 0.f;
            if (!q_finite && valid) set_status(p.status, MOE_ERR_NONFINITE);

            // ---- exchange: every thread merges the four lists in the same order ----
#pragma unroll
            for (int j = 0; j < kRTopK; ++j) s_ex[(c * kExWords + j) * 32 + lane] = qt[j];
            s_ex[(c * kExWords + kRTopK) * 32 + lane] = ssum;
            s_ex[(c * kExWords + kRTopK + 1) * 32 + lane] = q_finite ? 1.f : 0.f;
            named_bar(bar_id, 128);
            float l0[kRTopK], l1[kRTopK], sq[4];
            bool row_finite = true;
#pragma unroll
            for (int j = 0; j < kRTopK; ++j) {
                l0[j] = s_ex[(0 * kExWords + j) * 32 + lane];
                l1[j] = s_ex[(1 * kExWords + j) * 32 + lane];
            }
            merge8_desc(l0, l1);
            float l2[kRTopK], l3[kRTopK];
#pragma unroll
            for (int j = 0; j < kRTopK; ++j) {
                l2[j] = s_ex[(2 * kExWords + j) * 32 + lane];
                l3[j] = s_ex[(3 * kExWords + j) * 32 + lane];
            }
            merge8_desc(l2, l3);
            float qmax[4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                qmax[cc] = s_ex[(cc * kExWords + 0) * 32 + lane];
                sq[cc] = s_ex[(cc * kExWords + kRTopK) * 32 + lane];
                row_finite = row_finite && s_ex[(cc * kExWords + kRTopK + 1) * 32 + lane] != 0.f;
            }
            merge8_desc(l0, l2);  // l0: the token's eight largest scores
            named_bar(bar_id, 128);  // the exchange area becomes the candidate slots
            const float tau = l0[kRTopK - 1];
            const float mx = l0[0];
            const float mxL = mx * kLog2e;
            float den = 0.f;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) den += sq[cc] * ex2_approx(fmaf(qmax[cc], kLog2e, -mxL));
            // p = 2^(s log2e - (max log2e + log2 den)); rows outside the run or with a
            // non-finite score contribute nothing to the probability sums
            const float cL = mxL + log2f(den);
            const float pcap = (valid && row_finite) ? INFINITY : 0.f;

            // ---- pass 2: probabilities and the candidates ----
            uint32_t slot = slot_base;
            uint32_t eq_bits[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t r[32];
                tmem_ld32(tcol + 32 * h, r);
                tmem_ld_wait(r);
                float pr[32];
                uint32_t eqb = 0;
                const float4* b4 = reinterpret_cast<const float4*>(s_bias + c * CQ + 32 * h);
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const float4 b = b4[j4];
                    const float bb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int j = 4 * j4 + u;
                        const float xv = __uint_as_float(r[j]) + bb[u];
                        pr[j] = fminf(ex2_approx(fmaf(xv, kLog2e, -cL)), pcap);  // fminf drops a NaN
                        // a score above tau goes to the next slot; one equal to tau sets its bit
                        if (xv > tau && slot <= slot_last) {  // seven at most; the bound only guards the area
                            asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(slot), "f"(xv),
                                         "f"(__int_as_float(c * CQ + 32 * h + j)));
                            slot += 1024u;
                        }
                        eqb |= xv == tau ? (1u << j) : 0u;
                    }
                }
                eq_bits[h] = eqb;
                const float cs = transpose_sum32(pr, lane);
                acc_ps[h] += cs;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_l + 8u * acc);  // the next tile may use the accumulator

            // ---- select: the quarter's candidates in (score desc, index asc) order ----
            float tv[kRTopK];
            int ti[kRTopK];
#pragma unroll
            for (int j = 0; j < kRTopK; ++j) {
                tv[j] = -INFINITY;
                ti[j] = c * CQ + j;
            }
            const int n_gt = (int)((slot - slot_base) >> 10);  // <= kSlots
            for (int s = 0; s < n_gt; ++s) {
                float2 e;
                asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(e.x), "=f"(e.y) : "r"(slot_base + 1024u * (uint32_t)s));
                topk_insert(tv, ti, e.x, __float_as_int(e.y));
            }
            // the experts tied at tau, ascending; no list needs more than eight of them
#pragma unroll 1
            for (int h = 0, n_eq = 0; h < 2; ++h) {
                uint32_t b = eq_bits[h];
                while (b != 0u && n_eq < kRTopK) {
                    const int j = __ffs(b) - 1;
                    b &= b - 1u;
                    topk_insert(tv, ti, tau, c * CQ + 32 * h + j);
                    ++n_eq;
                }
            }

            // ---- merge the four lists: (1 into 0, 3 into 2), then (2 into 0) ----
            if (c & 1) {
#pragma unroll
                for (int j = 0; j < kRTopK; ++j) {
                    s_mv[((c >> 1) * kRTopK + j) * 32 + lane] = tv[j];
                    s_mi[((c >> 1) * kRTopK + j) * 32 + lane] = ti[j];
                }
            }
            named_bar(bar_id, 128);
            // a list holds its candidates first and fillers of -inf after them: insert up to the first
            // filler (a row whose top-8 reaches -inf has a non-finite score and is flagged)
            if (!(c & 1)) {
#pragma unroll 1
                for (int j = 0; j < kRTopK; ++j) {
                    const float v = s_mv[((c >> 1) * kRTopK + j) * 32 + lane];
                    if (!(v > -INFINITY)) break;
                    topk_insert(tv, ti, v, s_mi[((c >> 1) * kRTopK + j) * 32 + lane]);
                }
            }
            if (c == 2) {  // list 1 was read by this thread only
#pragma unroll
                for (int j = 0; j < kRTopK; ++j) {
                    s_mv[(kRTopK + j) * 32 + lane] = tv[j];
                    s_mi[(kRTopK + j) * 32 + lane] = ti[j];
                }
            }
            named_bar(bar_id, 128);
            if (c == 0) {
#pragma unroll 1
                for (int j = 0; j < kRTopK; ++j) {
                    const float v = s_mv[(kRTopK + j) * 32 + lane];
                    if (!(v > -INFINITY)) break;
                    topk_insert(tv, ti, v, s_mi[(kRTopK + j) * 32 + lane]);
                }
                if (write) {
                    // gates: softmax of the selected scores (the first is the largest)
                    float ex[kRTopK];
                    float es = 0.f;
#pragma unroll
                    for (int j = 0; j < kRTopK; ++j) {
                        ex[j] = j < p.k ? __expf(tv[j] - tv[0]) : 0.f;
                        es += ex[j];
                    }
                    const float ginv = 1.0f / es;
#pragma unroll
                    for (int j = 0; j < kRTopK; ++j) {
                        if (j < p.k) {
                            const float g = ex[j] * ginv;
                            p.selected[t * p.k + j] = (int64_t)ti[j];
                            atomicAdd(&s_counts[ti[j]], 1);
                            if (p.gates_f32) p.gates_f32[t * p.k + j] = g;
                            if (p.gates) {
                                if (p.gates_bf16)
                                    reinterpret_cast<__nv_bfloat16*>(p.gates)[t * p.k + j] = __float2bfloat16_rn(g);
                                else
                                    reinterpret_cast<float*>(p.gates)[t * p.k + j] = g;
                            }
                        }
                    }
                }
            }
        }
        // per-CTA partials: the four lane quarters of each expert in a fixed order
        named_bar(5, kREpiWarps * 32);  // every group is done with its union area
        float* s_psum = reinterpret_cast<float*>(smem_raw + kOffUnion);  // [q][E]
#pragma unroll
        for (int h = 0; h < 2; ++h) s_psum[q * E + c * CQ + 32 * h + lane] = acc_ps[h];
        named_bar(5, kREpiWarps * 32);
        for (int e = threadIdx.x - 96; e < E; e += kREpiWarps * 32) {
            p.part_psum[(int64_t)blockIdx.x * E + e] =
                ((s_psum[0 * E + e] + s_psum[1 * E + e]) + s_psum[2 * E + e]) + s_psum[3 * E + e];
            p.part_counts[(int64_t)blockIdx.x * E + e] = s_counts[e];
        }
    }

    tc_fence_before();
    cluster_sync();  // neither CTA leaves while the other may still signal its barriers or read its stages
    if (warp == 2) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(2 * E) : "memory");
    }
}

int launch_fused(const CUtensorMap& mx, const CUtensorMap& mw, const RFParams& rp, int grid, cudaStream_t stream) {
    static bool attr_set[64] = {false};
    int dev = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 64 && !attr_set[dev]) {
        MOE_CUDA_TRY(cudaFuncSetAttribute(route_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)kSmemBytes));
        attr_set[dev] = true;
    }
    route_fused_kernel<<<grid, kRThreads, kSmemBytes, stream>>>(mx, mw, rp);
    return launch_status();
}

}  // namespace

bool route_fused_supported(int64_t T, int64_t D, int64_t ldx, const void* x, const void* w_ed, int32_t E,
                           int32_t k) {
    return E == 256 && k >= 1 && k <= kRTopK && D >= 1 && D % 8 == 0 && ldx % 8 == 0 &&
           aligned16(x) && aligned16(w_ed) && T >= 1 && T < (int64_t(1) << 31);
}

int route_fused_grid(int64_t T) {
    const int64_t units = (T + kRBox - 1) / kRBox;
    const int64_t pairs = device_sm_count() / 2;
    return 2 * (int)(units < pairs ? units : pairs);
}

int route_fused_run(const void* x, int64_t T, int64_t D, int64_t ldx, const void* w_ed, int32_t E,
                    const float* bias, int32_t k, float* logits_out, int64_t* selected, void* gates, int gates_bf16,
                    float* gates_f32, int32_t* part_counts, float* part_psum, int32_t* status, cudaStream_t stream) {
    MOE_REQUIRE(route_fused_supported(T, D, ldx, x, w_ed, E, k), MOE_ERR_UNSUPPORTED);
    CUtensorMap mx, mw;
    MOE_REQUIRE(make_map(&mx, x, D, T, ldx, kRBox), MOE_ERR_CUDA);
    MOE_REQUIRE(make_map(&mw, w_ed, D, E, D, E / 2), MOE_ERR_CUDA);
    RFParams rp{};
    rp.T = T;
    rp.units = (T + kRBox - 1) / kRBox;
    rp.k = k;
    rp.k_blocks = (int)((D + kRBK - 1) / kRBK);
    rp.bias = bias;
    rp.logits_out = logits_out;
    rp.selected = selected;
    rp.gates = gates;
    rp.gates_bf16 = gates_bf16;
    rp.gates_f32 = gates_f32;
    rp.part_counts = part_counts;
    rp.part_psum = part_psum;
    rp.status = status;
    const int grid = route_fused_grid(T);
    return launch_fused(mx, mw, rp, grid, stream);
}

}  // namespace moe
