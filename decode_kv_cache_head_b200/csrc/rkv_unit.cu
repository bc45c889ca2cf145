// rkv_unit.cu -- the R-KV compression step with one CTA per unit (sequence,
// layer, KV head), for launches with at least as many units as the GPU has
// SMs: no cluster, no exchange, one select per unit.
//
// Method: "R-KV: Redundancy-aware KV Cache Compression for Reasoning Models"
// (atlas.scime.ai summary, "Approach": Z = lambda I - (1 - lambda) R, applied
// periodically during decoding; "Measured effects": max pooling over the GQA
// group), the hysenlabs write-up (decode-time scoring: budget, window_size,
// mix_lambda; the protected recent window) and the sourcepulse summary ("How
// It Works": attention-weight importance, cosine-similarity redundancy, top-k
// within the budget).
//
// A unit's K (N rows x 256 bytes) is larger than shared memory, so it is
// streamed twice through a two-stage ring of 128-row tiles loaded by TMA:
//   pass 1 (from HBM): one thread issues tcgen05 UMMAs, logits[128 rows, G*w]
//     = K_tile . Q^T into TMEM; meanwhile the CTA computes ||k_i||^2 and
//     1/max(||k_i||, 1e-12) and its running part of S = sum_i khat_i; then
//     every thread folds its row's logits into per-column running (max, sum
//     of exp) pairs (online softmax, rescaling only when a logit exceeds the
//     running reference by more than 2^8).
//   between the passes: the column pairs are merged over the CTA; S is split
//     into three bf16 terms (hi + mid + lo carries its fp32 value) and written
//     as three extra rows of the UMMA B operand.
//   pass 2 (the same tiles, last to first, now from L2): the UMMA gives the logits again and,
//     in three more columns, k_i . S; per row p = exp(s - max) / sum, the mean
//     over the window queries and the max over the group (Ihat_i), and
//     r_i = (khat_i . S - khat_i . khat_i) / (N - 1) (MEAN) or r_i from the
//     similarity kernel (MAX).
//   then the normalisers, the joint scores, the radix select and the
//   destinations of the kept rows, and the in-place compaction of K, then of V,
//   in ascending chunks of 128 rows (every source row of a chunk is read before
//   any row of it is written; later chunks only read rows above the current
//   chunk, so the next chunk's reads overlap this chunk's writes).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cfloat>
#include <cstdint>
#include <type_traits>

#include "rkv_block.cuh"
#include "rkv_internal.h"
#include "rkv_post.cuh"
#include "rkv_ptx.cuh"

namespace rkv {

namespace {

constexpr int kTileRows = 128;
constexpr uint32_t kStageBytes = 32768u;
constexpr uint32_t kHalfBytes = 16384u;
constexpr int kChunkRows = 128;          // compaction chunk of one tensor (two in flight)
constexpr float kRescaleLog2 = 8.0f;     // online softmax: rescale past 2^8

// Merges (m2, s2) into (m, s): s = sum of 2^(x - m) over the values seen.
__device__ __forceinline__ void ms_merge(float &m, float &s, float m2, float s2) {
    const float mn = fmaxf(m, m2);
    const float a = (m == -INFINITY) ? 0.f : s * ex2_approx(m - mn);
    const float b = (m2 == -INFINITY) ? 0.f : s2 * ex2_approx(m2 - mn);
    m = mn;
    s = a + b;
}

// Folds 8 per-lane columns of (m, s) pairs across the warp: afterwards lane L
// holds the merge over all 32 lanes of column (L & 7) in m[0], s[0].
__device__ __forceinline__ void warp_fold8_ms(float (&m)[8], float (&s)[8]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1) {
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send_m = up ? m[i] : m[i + off];
            const float send_s = up ? s[i] : s[i + off];
            float km = up ? m[i + off] : m[i];
            float ks = up ? s[i + off] : s[i];
            const float rm = __shfl_xor_sync(kFull, send_m, off);
            const float rs = __shfl_xor_sync(kFull, send_s, off);
            ms_merge(km, ks, rm, rs);
            m[i] = km;
            s[i] = ks;
        }
    }
#pragma unroll
    for (int off = 8; off <= 16; off <<= 1) {
        const float rm = __shfl_xor_sync(kFull, m[0], off);
        const float rs = __shfl_xor_sync(kFull, s[0], off);
        ms_merge(m[0], s[0], rm, rs);
    }
}

__device__ __forceinline__ uint16_t bf16_rn_bits(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

}  // namespace

// NQP: query columns G*w rounded up to 16.  WC: the window when it is 8 (the
// pages' value), 0 for a runtime window.
template <int NQP, int WC>
__global__ void __launch_bounds__(kUnitThreads, 2) rkv_unit_kernel(const __grid_constant__ UnitParams p) {
    constexpr int NT = kUnitThreads;
    constexpr int NW = NT / 32;
    constexpr int SLOT = NQP + 16;          // TMEM columns per tile slot
    constexpr int HC = NQP / 2;             // pass-1 columns per warpgroup
    constexpr uint32_t kBRows = NQP + 16;   // B operand rows: queries, then the split S
    constexpr int MAXH = NQP / 16;          // heads per warpgroup in pass 2 (WC == 8)
    static_assert(WC == 0 || WC == 8, "window template");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wg = warp >> 2;

    // launched as a programmatic dependent of the plan kernel: nothing it wrote (or that
    // ran before it) is read before this wait
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const UnitCoord uc = unit_coord(static_cast<int>(blockIdx.x), p.n_kv, p.batch,
                                    static_cast<int>(gridDim.x) / (p.n_kv * p.batch), p.order);
    const int h = uc.h, b = uc.b, l = uc.l;
    const int N = p.n_eff[b];
    if (N <= 0) return;   // not due

    const int w = WC > 0 ? WC : p.window;
    const int G = p.group;
    const int NQ = G * w;
    const int M = N - w;
    const int budget = p.budgets ? p.budgets[b] : p.budget_cfg;
    const float lam = p.lambdas ? p.lambdas[b] : p.lambda_cfg;
    const int kk = budget - w;
    const bool red_max = p.red_mode == RKV_RED_MAX;
    const bool pool_max = p.gqa_pool == RKV_GQA_MAX;
    const int T = (N + kTileRows - 1) / kTileRows;
    const int64_t krow0 = unit_first_row(p.seq_row, p.seq_cap, b, h, p.n_kv, p.cap);
    // paged caches: row r of this unit is row prow(r) of the layer's page pool
    const bool paged = p.block_table != nullptr;
    const int psh = paged ? 31 - __clz(p.page_rows) : 7;   // page_rows is a power of two
    const int P = 1 << psh;
    const int64_t unit_g = (static_cast<int64_t>(p.layer_base + l) * p.batch + b) * p.n_kv + h;

    const UnitLayout L = make_unit_layout(p.nmax, NQP);
    uint8_t *sStage = base + L.stage;
    uint8_t *sB = base + L.b;
    float *sSS = reinterpret_cast<float *>(base + L.ss);       // ||k_i||^2 (pass 1 -> pass 2)
    float *sIhat = reinterpret_cast<float *>(base + L.ihat);   // Ihat (max or sum over heads)
    float *sR = reinterpret_cast<float *>(base + L.r);
    float *sScr = reinterpret_cast<float *>(base + L.scr);
    float *sColM = reinterpret_cast<float *>(base + L.colm);
    float *sColF = reinterpret_cast<float *>(base + L.colf);
    uint64_t *sVis = reinterpret_cast<uint64_t *>(base + L.vis);
    float *sRed = reinterpret_cast<float *>(base + L.red);
    uint32_t *sRedU = reinterpret_cast<uint32_t *>(base + L.red);
    // full[2] (TMA), mma[2] (logits UMMA), smma[2] (S UMMA); then the TMEM base and
    // the per-stage count of warps whose S-UMMA operand is written
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + L.bars);
    uint32_t *sTmem = reinterpret_cast<uint32_t *>(bars + 6);
    uint32_t *sBsCount = sTmem + 2;
    // after the last tile the ring holds the keys, the destinations and the histograms
    const uint32_t arr = align_up(static_cast<uint32_t>(p.nmax) * 4u, 16);
    uint32_t *sKeys = reinterpret_cast<uint32_t *>(sStage);
    int32_t *sDst = reinterpret_cast<int32_t *>(sStage + arr);
    uint32_t *sHist = reinterpret_cast<uint32_t *>(sStage + 2u * arr);
    int32_t *sBT = reinterpret_cast<int32_t *>(base + L.bt);
    auto prow = [&](int r) -> int64_t {   // row of the layer's 2-D view holding unit row r
        return paged ? ((static_cast<int64_t>(sBT[r >> psh]) * p.n_kv + h) << psh) + (r & (P - 1))
                     : krow0 + r;
    };

    const uint64_t colmask = NQ >= 64 ? ~0ull : ((1ull << NQ) - 1ull);
    const uint64_t lastmask = [&] {
        uint64_t m = 0;
        for (int g = 0; g < G; ++g) m |= 1ull << (g * w + w - 1);
        return m;
    }();

    // ---- set-up
    uint8_t *sBs = base + L.bs;   // B operand of the S UMMA, two buffers of 16 rows x 128 tokens
    uint64_t *full = bars, *mmab = bars + 2, *smma = bars + 4;
    if (warp == 0) {
        tmem_alloc(sTmem, static_cast<uint32_t>(p.tmem_cols));
        tmem_relinquish();
    }
    if (tid == 32) {
        for (int i = 0; i < 6; ++i) mbar_init(&bars[i], 1);
        sBsCount[0] = sBsCount[1] = 0;
        fence_mbar_init();
    }
    // B operand rows past the queries start as zeros (the split S lands in three of
    // them), and so do both S-UMMA B buffers (rows 3..15 stay zero)
    for (int i = tid; i < 2 * 16 * 8; i += NT) {
        const int half = i >> 7, row = NQP + ((i & 127) >> 3), ch = i & 7;
        *reinterpret_cast<uint4 *>(sB + half * kBRows * 128u + row * 128u + ch * 16u) =
            make_uint4(0u, 0u, 0u, 0u);
    }
    for (int i = tid; i < 2 * 4096 / 16; i += NT)
        reinterpret_cast<uint4 *>(sBs)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (paged)
        for (int j = tid; j < (N + P - 1) / P; j += NT) sBT[j] = p.block_table[static_cast<int64_t>(b) * p.max_blocks + j];
    // window key M + d is seen by query column g*w + j only when j >= d (causal)
    if (warp == 0) {
        const int j0 = lane % w, j1 = (lane + 32) % w;
        for (int d = 0; d < w; ++d) {
            const uint64_t m =
                static_cast<uint64_t>(__ballot_sync(kFull, lane < NQ && j0 >= d)) |
                (static_cast<uint64_t>(__ballot_sync(kFull, lane + 32 < NQ && j1 >= d)) << 32);
            if (lane == 0) sVis[d] = m;
        }
    }
    fence_proxy_async_smem();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *sTmem;
    const uint32_t scol = static_cast<uint32_t>(2 * SLOT);   // S accumulator columns

    // last tile / logits UMMA / S UMMA issued (thread 0's copies), for the error path
    int tma_last = 1, mma_last = -1;
    const CUtensorMap *mk = &p.tmap_k[l];
    // global tile g: pass 1 takes tiles 0 .. T-1, pass 2 the same tiles from T-1 down to 0,
    // so it starts on the tiles pass 1 read last (the most likely still in L2) and ends on the
    // first ones, which the compaction reads first
    auto tile_of = [&](int g) { return g < T ? g : 2 * T - 1 - g; };
    auto issue_tile = [&](int g) {
        tma_last = g;
        const int tt = tile_of(g);
        uint8_t *stg = sStage + (g & 1) * kStageBytes;
        // K tiles are kept in L2 (evict last): pass 2 and the compaction read them again
        const uint64_t pol = policy_evict_last();
        if (!paged) {
            const int32_t y = static_cast<int32_t>(krow0 + tt * kTileRows);
            tma_load_2d_hint(stg, mk, &full[g & 1], 0, y, pol);
            tma_load_2d_hint(stg + kHalfBytes, mk, &full[g & 1], 64, y, pol);
        } else {
            // one box per page; pages past the sequence's last read as zeros (a row
            // coordinate below the pool)
            const int npg = (N + P - 1) / P;
            for (int j = 0; j < kTileRows / P; ++j) {
                const int pg = tt * (kTileRows / P) + j;
                const int32_t y = pg < npg ? static_cast<int32_t>(prow(pg * P)) : -P;
                tma_load_2d_hint(stg + j * P * 128, mk, &full[g & 1], 0, y, pol);
                tma_load_2d_hint(stg + kHalfBytes + j * P * 128, mk, &full[g & 1], 64, y, pol);
            }
        }
    };
    // logits (and in pass 2 of MEAN mode k . S) of tile g into TMEM slot g & 1
    auto issue_logits = [&](int g) {
        mma_last = g;
        tc_fence_after();
        const bool with_s = g >= T && !red_max;
        const uint32_t idesc = with_s ? idesc_bf16_f32(128, NQP + 16) : idesc_bf16_f32(128, NQP);
        // A: the tile's two 64-column halves 16 KB apart; B: the queries (and split S), halves
        // kBRows x 128 bytes apart; eight K steps issued from one asm block
        umma_bf16_k128_sw128<kBRows * 8u>(tmem_base + static_cast<uint32_t>((g & 1) * SLOT),
                                          desc_lo_sw128(smem_u32(sStage + (g & 1) * kStageBytes)),
                                          desc_lo_sw128(smem_u32(sB)), idesc);
        umma_commit(&mmab[g & 1]);
    };
    if (tid == 0) {
        const CUtensorMap *mq = &p.tmap_q[l];
        const int32_t yq = (b * p.n_kv + h) * NQ;   // the KV head's query rows
        mbar_arrive_expect_tx(&full[0], kStageBytes + static_cast<uint32_t>(NQP) * 256u);
        tma_load_2d(sB, mq, &full[0], 0, yq);
        tma_load_2d(sB + kBRows * 128u, mq, &full[0], 64, yq);
        issue_tile(0);
        mbar_arrive_expect_tx(&full[1], kStageBytes);
        issue_tile(1);
    }

    // ---- the two passes
    const float sc = p.logit_scale_log2;
    const float inv_nm1 = 1.0f / static_cast<float>(N - 1);
    const float inv_w = 1.0f / static_cast<float>(w);
    const uint32_t tmem_lane = tmem_base + ((32u * static_cast<uint32_t>(warp & 3)) << 16);
    const int lrow = (warp & 3) * 32 + lane;   // TMEM lane = tile row
    // norms: lanes 0-7 / 16-23 take the first 64 columns of rows (l & 7) + 8 (l >> 4)
    const int nrow = (lane & 7) + 8 * (lane >> 4), nhalf = (lane >> 3) & 1;
    const int row_t = 16 * warp + nrow;        // this lane's tile row in the norms

    // pass-1 column pairs of this warpgroup's HC columns, two columns per float2:
    // ncm = -(running reference), cs = sum of 2^(x - reference)
    float2 ncm[HC / 2], cs[HC / 2];
#pragma unroll
    for (int c = 0; c < HC / 2; ++c) {
        ncm[c] = make_float2(INFINITY, INFINITY);
        cs[c] = make_float2(0.f, 0.f);
    }
    const float2 sc2 = make_float2(p.logit_scale_log2, p.logit_scale_log2);
    bool ok = true;
    int g = 0;
    for (; g < 2 * T; ++g) {
        const bool pass2 = g >= T;
        const int tt = tile_of(g);
        const int s = g & 1;
        const uint32_t par = static_cast<uint32_t>((g >> 1) & 1);
        uint8_t *stg = sStage + s * kStageBytes;
        const uint32_t tslot = static_cast<uint32_t>(s * SLOT);
        bool wait_ok = true;

        if (!pass2) {
            wait_ok = mbar_wait(&full[s], par);
            if (tid == 0 && wait_ok) issue_logits(g);
            if (!red_max) {
                if (wait_ok) {
                    // ||k_i||^2 and 1 / max(||k_i||, 1e-12): two lanes per row, 64 columns each
                    const int i = tt * kTileRows + row_t;
                    const uint8_t *hp = stg + nhalf * kHalfBytes + row_t * 128;
                    float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 raw = *reinterpret_cast<const uint4 *>(hp + ((c ^ (row_t & 7)) << 4));
                        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(h2[e]);
                            ss2 = __ffma2_rn(f, f, ss2);
                        }
                    }
                    const float ssh = ss2.x + ss2.y;
                    const float ss = ssh + __shfl_xor_sync(kFull, ssh, 8);
                    const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
                    if (nhalf == 0) {
                        // inv as hi + mid + lo bf16: column row_t of the S-UMMA B operand
                        const bool in = i < N;
                        const uint16_t hi = in ? bf16_rn_bits(inv) : 0;
                        const float r1 = inv - bf16_bits_to_float(hi);
                        const uint16_t mid = in ? bf16_rn_bits(r1) : 0;
                        const uint16_t lo = in ? bf16_rn_bits(r1 - bf16_bits_to_float(mid)) : 0;
                        uint8_t *bb = sBs + s * 4096 + (row_t >> 6) * 2048;
                        const uint32_t c = (row_t & 63) >> 3, e = (row_t & 7) * 2u;
                        *reinterpret_cast<uint16_t *>(bb + sw128_offset(0, c) + e) = hi;
                        *reinterpret_cast<uint16_t *>(bb + sw128_offset(1, c) + e) = mid;
                        *reinterpret_cast<uint16_t *>(bb + sw128_offset(2, c) + e) = lo;
                        if (in) sSS[i] = ss;
                    }
                }
                if (tt == T - 1 && N < T * kTileRows) {
                    // rows past N (stale cache memory) become zeros before the S UMMA
                    // sums over them; the logits UMMA has finished reading them
                    wait_ok = wait_ok && mbar_wait(&mmab[s], par);
                    const int nv = N - tt * kTileRows;
                    for (int idx = tid; idx < (kTileRows - nv) * 16; idx += NT) {
                        const int r = nv + (idx >> 4), c = idx & 15;
                        *reinterpret_cast<uint4 *>(stg + (c >> 3) * kHalfBytes + r * 128 + ((c & 7) << 4)) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                // each warp's S-operand (and tail) writes, then a count: the warp that
                // completes it issues the S UMMA, so no warp waits for the others here
                fence_proxy_async_smem();
                __syncwarp();
                uint32_t last = 0;
                if (lane == 0) {
                    __threadfence_block();
                    last = atomicAdd(&sBsCount[s], 1u) == NW - 1 ? 1u : 0u;
                }
                last = __shfl_sync(kFull, last, 0);
                if (last && lane == 0) {
                    __threadfence_block();
                    sBsCount[s] = 0;   // the stage's next pass-1 tile counts from zero
                    // S += K_tile^T . inv: A = the K tile read MN-major (M = 128 columns,
                    // 64-column blocks 16 KB apart, 8-row groups 1 KB apart), B = inv split
                    tc_fence_after();
                    constexpr uint32_t idesc_s = idesc_bf16_f32_amn(128, 16);
                    // A MN-major: K steps of 16 rows are 2 KB apart; B: 64-row halves 2 KB apart
                    const uint32_t a_lo = static_cast<uint32_t>(desc_mnmajor_sw128(smem_u32(stg), kHalfBytes, 1024u));
                    umma_bf16_k128<128u, 512u, 128u>(tmem_base + scol, a_lo,
                                                     desc_lo_sw128(smem_u32(sBs + s * 4096)), idesc_s,
                                                     g > 0 ? 1u : 0u);
                    umma_commit(&smma[s]);
                }
            }
        } else if (g == T) {
            // ---- between the passes: column (max, sum) over the CTA; S split into B
            float *xm = sScr;   // [8 warps][HC] (m, s) pairs
#pragma unroll
            for (int c0 = 0; c0 < HC; c0 += 8) {
                float m8[8], s8[8];
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    m8[j] = -ncm[(c0 + j) / 2].x;
                    m8[j + 1] = -ncm[(c0 + j) / 2].y;
                    s8[j] = cs[(c0 + j) / 2].x;
                    s8[j + 1] = cs[(c0 + j) / 2].y;
                }
                warp_fold8_ms(m8, s8);
                if (lane < 8) {
                    xm[(warp * HC + c0 + lane) * 2] = m8[0];
                    xm[(warp * HC + c0 + lane) * 2 + 1] = s8[0];
                }
            }
            if (!red_max) {
                wait_ok = mbar_wait(&smma[(T - 1) & 1], static_cast<uint32_t>(((T - 1) >> 1) & 1));
                tc_fence_after();
                if (warp < 4 && wait_ok) {
                    uint32_t sv[4];
                    tmem_ld4_nowait(tmem_lane + scol, sv);
                    tmem_wait_ld();
                    reg_tie4(sv);
                    const float S = (__uint_as_float(sv[0]) + __uint_as_float(sv[1])) + __uint_as_float(sv[2]);
                    const int d = 32 * warp + lane;
                    const uint16_t hi = bf16_rn_bits(S);
                    const float r1 = S - bf16_bits_to_float(hi);
                    const uint16_t mid = bf16_rn_bits(r1);
                    const uint16_t lo = bf16_rn_bits(r1 - bf16_bits_to_float(mid));
                    uint8_t *hb = sB + (d >> 6) * kBRows * 128u;
                    const uint32_t c = (d & 63) >> 3, e = (d & 7) * 2u;
                    *reinterpret_cast<uint16_t *>(hb + sw128_offset(NQP + 0, c) + e) = hi;
                    *reinterpret_cast<uint16_t *>(hb + sw128_offset(NQP + 1, c) + e) = mid;
                    *reinterpret_cast<uint16_t *>(hb + sw128_offset(NQP + 2, c) + e) = lo;
                }
            }
            __syncthreads();
            if (tid < NQP) {
                const int q = tid, gq = q / HC, c = q % HC;
                float m = xm[((gq * 4) * HC + c) * 2], sm = xm[((gq * 4) * HC + c) * 2 + 1];
#pragma unroll
                for (int k = 1; k < 4; ++k)
                    ms_merge(m, sm, xm[((gq * 4 + k) * HC + c) * 2], xm[((gq * 4 + k) * HC + c) * 2 + 1]);
                sColM[q] = -m;   // negated: pass 2 adds it
                sColF[q] = sm > 0.f ? 1.0f / sm : 0.f;
            }
            // Ihat starts at zero: both warpgroups merge their heads into it in pass 2
            // (the S UMMA that read these bytes is complete)
            for (int j = tid; j < M; j += NT) sIhat[j] = 0.f;
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0 && wait_ok) {
                if (mbar_wait(&full[s], par)) issue_logits(g);
            }
        }

        wait_ok = wait_ok && mbar_wait(&mmab[s], par);
        tc_fence_after();
        const int i = tt * kTileRows + lrow;
        if (wait_ok && !pass2) {
            // ---- pass 1: fold this row's logits into the running column pairs
            const uint64_t rmask = i < M ? colmask : (i < N ? sVis[i - M] : 0ull);
            const bool all_cand = __all_sync(kFull, i < M);
            // up to 16 columns: all loads in flight at once; more: one 8-column load at a time
            constexpr int NB = HC <= 16 ? HC / 8 : 1;
            uint32_t raw[NB][8];
            if (HC <= 16) {
#pragma unroll
                for (int c0 = 0; c0 < HC; c0 += 8)
                    tmem_ld8_nowait(tmem_lane + tslot + static_cast<uint32_t>(wg * HC + c0), raw[(c0 / 8) % NB]);
                tmem_wait_ld();
#pragma unroll
                for (int c0 = 0; c0 < HC; c0 += 8) reg_tie8(raw[(c0 / 8) % NB]);
            }
#pragma unroll
            for (int c0 = 0; c0 < HC; c0 += 8) {
                const int q0 = wg * HC + c0;
                if (HC > 16) {
                    tmem_ld8_nowait(tmem_lane + tslot + static_cast<uint32_t>(q0), raw[0]);
                    tmem_wait_ld();
                    reg_tie8(raw[0]);
                }
                const bool allv = all_cand && q0 + 8 <= NQ;   // warp-uniform
                float2 x[4], d[4];
                bool big = false;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    x[j] = __fmul2_rn(make_float2(__uint_as_float(raw[(c0 / 8) % NB][2 * j]),
                                                  __uint_as_float(raw[(c0 / 8) % NB][2 * j + 1])), sc2);
                    d[j] = __fadd2_rn(x[j], ncm[c0 / 2 + j]);   // x - reference
                }
                if (allv) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) big |= (d[j].x > kRescaleLog2) | (d[j].y > kRescaleLog2);
                    if (!__any_sync(kFull, big)) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            cs[c0 / 2 + j] = __fadd2_rn(cs[c0 / 2 + j],
                                                        make_float2(ex2_approx(d[j].x), ex2_approx(d[j].y)));
                        continue;
                    }
                }
                // masked columns or rows, or a logit past the rescale margin
                bool vis[8];
                big = false;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    vis[j] = allv || (((rmask >> (q0 + j)) & 1ull) != 0);
                    const float dj = (j & 1) ? d[j / 2].y : d[j / 2].x;
                    big |= vis[j] && (dj > kRescaleLog2);
                }
                if (__any_sync(kFull, big)) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if (vis[j]) {
                            float &nm = (j & 1) ? ncm[(c0 + j) / 2].y : ncm[(c0 + j) / 2].x;
                            float &sj = (j & 1) ? cs[(c0 + j) / 2].y : cs[(c0 + j) / 2].x;
                            const float xj = (j & 1) ? x[j / 2].y : x[j / 2].x;
                            const float mn = fmaxf(-nm, xj);
                            sj = sj * ex2_approx(-nm - mn) + ex2_approx(xj - mn);
                            nm = -mn;
                        }
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float dj = (j & 1) ? d[j / 2].y : d[j / 2].x;
                        float &sj = (j & 1) ? cs[(c0 + j) / 2].y : cs[(c0 + j) / 2].x;
                        const float e = ex2_approx(dj);
                        sj += vis[j] ? e : 0.f;
                    }
                }
            }
        } else if (wait_ok) {
            // ---- pass 2: Ihat partial (this warpgroup's heads) and r
            const bool cand = i < M;
            if (__any_sync(kFull, cand)) {
                float pool = 0.f;   // Ihat >= 0: 0 is neutral for both pools
                if (WC > 0) {
                    const int Ga = (G + 1) >> 1;
                    const int h0 = wg == 0 ? 0 : Ga, nh = wg == 0 ? Ga : G - Ga;
                    uint32_t raw[MAXH][8];
#pragma unroll
                    for (int k = 0; k < MAXH; ++k)
                        if (k < nh)
                            tmem_ld8_nowait(tmem_lane + tslot + static_cast<uint32_t>((h0 + k) * 8), raw[k]);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < MAXH; ++k)
                        if (k < nh) reg_tie8(raw[k]);
#pragma unroll
                    for (int k = 0; k < MAXH; ++k) {
                        if (k < nh) {
                            const int q0 = (h0 + k) * 8;
                            const float4 *nm4 = reinterpret_cast<const float4 *>(sColM + q0);
                            const float4 *f4 = reinterpret_cast<const float4 *>(sColF + q0);
                            float2 run2 = make_float2(0.f, 0.f);
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                const float4 nm = nm4[j], f = f4[j];
                                const float2 a0 = __ffma2_rn(make_float2(__uint_as_float(raw[k][4 * j]),
                                                                         __uint_as_float(raw[k][4 * j + 1])),
                                                             sc2, make_float2(nm.x, nm.y));
                                const float2 a1 = __ffma2_rn(make_float2(__uint_as_float(raw[k][4 * j + 2]),
                                                                         __uint_as_float(raw[k][4 * j + 3])),
                                                             sc2, make_float2(nm.z, nm.w));
                                run2 = __ffma2_rn(make_float2(ex2_approx(a0.x), ex2_approx(a0.y)),
                                                  make_float2(f.x, f.y), run2);
                                run2 = __ffma2_rn(make_float2(ex2_approx(a1.x), ex2_approx(a1.y)),
                                                  make_float2(f.z, f.w), run2);
                            }
                            const float a = (run2.x + run2.y) * inv_w;
                            pool = pool_max ? fmaxf(pool, a) : pool + a;
                        }
                    }
                } else if (wg == 0) {
                    uint32_t raw[NQP / 8][8];
#pragma unroll
                    for (int c0 = 0; c0 < NQP; c0 += 8)
                        tmem_ld8_nowait(tmem_lane + tslot + static_cast<uint32_t>(c0), raw[c0 / 8]);
                    tmem_wait_ld();
#pragma unroll
                    for (int c0 = 0; c0 < NQP; c0 += 8) reg_tie8(raw[c0 / 8]);
                    float run = 0.f;
#pragma unroll
                    for (int q = 0; q < NQP; ++q) {
                        if (q < NQ) {
                            run = fmaf(ex2_approx(fmaf(__uint_as_float(raw[q / 8][q % 8]), sc, sColM[q])),
                                       sColF[q], run);
                            if ((lastmask >> q) & 1ull) {
                                const float a = run * inv_w;
                                pool = pool_max ? fmaxf(pool, a) : pool + a;
                                run = 0.f;
                            }
                        }
                    }
                }
                float r = 0.f;
                if (wg == 1) {
                    if (red_max) {
                        r = cand ? p.r_ext[unit_g * p.cap + i] : 0.f;
                    } else {
                        uint32_t d[4];
                        tmem_ld4_nowait(tmem_lane + tslot + static_cast<uint32_t>(NQP), d);
                        tmem_wait_ld();
                        reg_tie4(d);
                        const float dot = (__uint_as_float(d[0]) + __uint_as_float(d[1])) + __uint_as_float(d[2]);
                        if (cand) {
                            // the inverse norm and khat_i . khat_i exactly as pass 1 had them
                            const float ss = sSS[i];
                            const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
                            const float self = __fmul_rn(__fmul_rn(inv, inv), ss);
                            r = (inv * dot - self) * inv_nm1;
                        }
                    }
                }
                if (cand) {
                    // pool >= 0, so its bits order like the value: the max of the two
                    // warpgroups' heads is an integer max; the mean pool adds two terms
                    // (a + b == b + a, whichever lands first)
                    if (pool_max)
                        atomicMax(reinterpret_cast<int *>(&sIhat[i]), __float_as_int(pool));
                    else
                        atomicAdd(&sIhat[i], pool);
                    if (wg == 1) sR[i] = r;
                }
            }
        }
        tc_fence_before();
        if (__syncthreads_or(!wait_ok || !ok)) {
            ok = false;
            break;
        }
        if (tid == 0) {
            // stage s is free once every UMMA reading it is done: the logits one
            // (waited above by everyone) and, in pass 1, the S one
            if (g + 2 < 2 * T) {
                if (pass2 || red_max || mbar_wait(&smma[s], par)) {
                    mbar_arrive_expect_tx(&full[s], kStageBytes);
                    issue_tile(g + 2);
                } else {
                    ok = false;
                }
            }
            // pass 2: the next tile's UMMA now, so that it runs during this warp's wait
            if (pass2 && ok && g + 1 < 2 * T) {
                if (mbar_wait(&full[(g + 1) & 1], static_cast<uint32_t>(((g + 1) >> 1) & 1)))
                    issue_logits(g + 1);
                else
                    ok = false;
            }
        }
    }
    // a wait of thread 0 after the last barrier of the loop
    if (__syncthreads_or(!ok)) ok = false;

    if (!ok) {
        // A wait ran out: record it, wait (bounded) for this CTA's copies and
        // UMMAs still in flight, free TMEM and leave without writing anything.
        if (tid == 0) {
            record_flag(p.status, kDevFlagTimeout);
            for (int gg = g; gg <= tma_last; ++gg)
                (void)mbar_wait(&full[gg & 1], static_cast<uint32_t>((gg >> 1) & 1));
            for (int gg = g; gg <= mma_last; ++gg)
                (void)mbar_wait(&mmab[gg & 1], static_cast<uint32_t>((gg >> 1) & 1));
            // the S UMMA of a pass-1 tile may come from any warp: wait for this one's
            if (g < T && !red_max) (void)mbar_wait(&smma[g & 1], static_cast<uint32_t>((g >> 1) & 1));
        }
        __syncthreads();
        if (warp == 0) {
            tc_fence_after();
            tmem_dealloc(tmem_base, static_cast<uint32_t>(p.tmem_cols));
        }
        return;
    }

    // ---- normalisers, keys and the select (one per unit)
    float inv_sumI, rmax_g, inv_rsum;
    uint32_t Tk = 0xffffffffu;
    int n_gt = 0;
    const float invG = 1.0f / static_cast<float>(G);
    const bool scores_only = p.z_heads != nullptr;
    post_scores_any<NT, 1>(
        [&](int j) { return make_float2(pool_max ? sIhat[j] : sIhat[j] * invG, sR[j]); },
        sKeys, sHist, sRed, M, kk, lam, !scores_only, inv_sumI, rmax_g, inv_rsum, Tk, n_gt);

    if (scores_only) {
        // shared selection: this head's joint score of every candidate; the
        // heads (and ranks) are summed and one set is selected afterwards
        float *zo = p.z_heads + unit_g * p.cap;
        for (int row = tid; row < M; row += NT) {
            const float I = (pool_max ? sIhat[row] : sIhat[row] * invG) * inv_sumI;
            const float Rv = ex2_approx((sR[row] - rmax_g) * kLog2e) * inv_rsum;
            zo[row] = joint_score(lam, I, Rv);
        }
        __syncthreads();
        if (warp == 0) {
            tc_fence_after();
            tmem_dealloc(tmem_base, static_cast<uint32_t>(p.tmem_cols));
        }
        return;
    }

    // ---- destination of every row: G_i = rows above the threshold or in the
    // window before i, E_i = tied candidates before i;
    // kept = above || window || (tied && E_i < need_eq), dst = G_i + min(E_i, need_eq)
    const int need_eq = (kk > 0) ? kk - n_gt : 0;
    {
        // warp w owns rows [w*seg, w*seg + seg): count, one block exchange of the
        // eight warp totals, then each warp walks its rows 32 at a time with ballots
        const int seg = ((N + NW - 1) / NW + 31) / 32 * 32;
        const int r0 = warp * seg, r1 = min(N, r0 + seg);
        const uint32_t lt = (1u << lane) - 1u;
        auto flags = [&](int row, bool &eq, bool &gw) {
            const bool in = row < r1;
            const bool cand = row < M;
            const uint32_t key = (in && cand) ? sKeys[row] : 0u;
            eq = in && cand && kk > 0 && key == Tk;
            gw = in && (!cand || (kk > 0 && key > Tk));
        };
        uint32_t ng = 0, ne = 0;
        for (int rb = r0; rb < r1; rb += 32) {
            bool eq, gw;
            flags(rb + lane, eq, gw);
            ng += __popc(__ballot_sync(kFull, gw));
            ne += __popc(__ballot_sync(kFull, eq));
        }
        if (lane == 0) {
            sRedU[warp] = ng;
            sRedU[NW + warp] = ne;
        }
        __syncthreads();
        uint32_t g_run = 0, e_run = 0;
        for (int w2 = 0; w2 < warp; ++w2) {
            g_run += sRedU[w2];
            e_run += sRedU[NW + w2];
        }
        for (int rb = r0; rb < r1; rb += 32) {
            bool eq, gw;
            const int row = rb + lane;
            flags(row, eq, gw);
            const uint32_t bg = __ballot_sync(kFull, gw), be = __ballot_sync(kFull, eq);
            const uint32_t Gi = g_run + __popc(bg & lt), Ei = e_run + __popc(be & lt);
            const bool kept = gw || (eq && Ei < static_cast<uint32_t>(need_eq));
            if (row < r1)
                sDst[row] = kept ? static_cast<int32_t>(Gi + min(Ei, static_cast<uint32_t>(need_eq))) : -1;
            g_run += __popc(bg);
            e_run += __popc(be);
        }
    }
    __syncthreads();

    if (p.kept_out || p.scores_out) {
        for (int row = tid; row < N; row += NT) {
            const int d = sDst[row];
            if (p.kept_out && d >= 0) p.kept_out[unit_g * p.cap + d] = row;
            if (p.scores_out && row < M) {
                float *so = p.scores_out + unit_g * 4 * p.cap;
                const float I = (pool_max ? sIhat[row] : sIhat[row] * invG) * inv_sumI;
                const float Rv = ex2_approx((sR[row] - rmax_g) * kLog2e) * inv_rsum;
                so[row] = I;
                so[p.cap + row] = sR[row];
                so[2 * p.cap + row] = Rv;
                so[3 * p.cap + row] = joint_score(lam, I, Rv);
            }
        }
    }

    // ---- compaction, in place, ascending chunks from the first row that moves
    {
        uint32_t first = static_cast<uint32_t>(N);
        for (int row = tid; row < N; row += NT)
            if (sDst[row] != row) {
                first = static_cast<uint32_t>(row);
                break;
            }
        first = __reduce_min_sync(kFull, first);
        if (lane == 0) sRedU[warp] = first;
        __syncthreads();
        first = sRedU[0];
#pragma unroll
        for (int k = 1; k < NW; ++k) first = min(first, sRedU[k]);
        // Software-pipelined: chunk c + 1 is read before chunk c is written.  Its
        // rows lie above every destination of chunk c, and every read of chunk c
        // precedes the barrier before chunk c's writes.  K is moved first, while the
        // rows the second pass just read are still in L2, then V.  The two cache
        // layouts are compiled separately so the contiguous one carries no page lookups.
        auto compaction = [&](auto paged_c, uint16_t *buf) {
            constexpr bool PG = decltype(paged_c)::value;
            auto row_of = [&](int r) -> int64_t {
                if constexpr (PG)
                    return ((static_cast<int64_t>(sBT[r >> psh]) * p.n_kv + h) << psh) + (r & (P - 1));
                else
                    return krow0 + r;
            };
            constexpr int PER = kChunkRows * 16 / NT;   // 16-byte pieces per thread per chunk
            auto load = [&](int c0, uint4 (&x)[PER], int (&dd)[PER]) {
#pragma unroll
                for (int k = 0; k < PER; ++k) {
                    const int idx = tid + k * NT;
                    const int row = c0 + (idx >> 4), pc = idx & 15;
                    const int d = row < N ? sDst[row] : -1;
                    dd[k] = (d >= 0 && d != row) ? d : -1;
                    if (dd[k] >= 0) x[k] = __ldcg(reinterpret_cast<const uint4 *>(buf + row_of(row) * kHeadDim) + pc);
                }
            };
            // streaming (evict-first) stores: the moved rows are not read again by this
            // step, so they leave L2 early instead of displacing the rows still to be read
            auto store = [&](const uint4 (&x)[PER], const int (&dd)[PER]) {
#pragma unroll
                for (int k = 0; k < PER; ++k) {
                    if (dd[k] >= 0) {
                        const int pc = (tid + k * NT) & 15;
                        __stcs(reinterpret_cast<uint4 *>(buf + row_of(dd[k]) * kHeadDim) + pc, x[k]);
                    }
                }
            };
            uint4 xa[PER], xc[PER];
            int da[PER], dc[PER];
            int c0 = static_cast<int>(first);
            if (c0 < N) load(c0, xa, da);
            while (c0 < N) {
                const int c1 = c0 + kChunkRows;
                if (c1 < N) load(c1, xc, dc);
                __syncthreads();
                store(xa, da);
                if (c1 >= N) break;
                const int c2 = c1 + kChunkRows;
                if (c2 < N) load(c2, xa, da);
                __syncthreads();
                store(xc, dc);
                c0 = c2;
            }
        };
        uint16_t *kb = p.k[l];
        uint16_t *vb = p.v[l];
        if (paged) {
            compaction(std::true_type{}, kb);
            compaction(std::true_type{}, vb);
        } else {
            compaction(std::false_type{}, kb);
            compaction(std::false_type{}, vb);
        }
    }

    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, static_cast<uint32_t>(p.tmem_cols));
    }
}

template <int NQP, int WC>
static cudaError_t launch_unit_t(const UnitParams &p, int n_units, size_t smem, cudaStream_t stream) {
    auto kern = rkv_unit_kernel<NQP, WC>;
    static std::atomic<int> granted{0};
    const cudaError_t e = ensure_smem_attr(kern, smem, granted);
    if (e != cudaSuccess) return e;
    // programmatic dependent launch: the CTAs may be scheduled while the preceding
    // kernel (the plan) finishes, and wait for it on the device
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_units), 1, 1);
    cfg.blockDim = dim3(kUnitThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

cudaError_t launch_unit(const UnitParams &p, int n_units, int nqp, size_t smem, cudaStream_t stream) {
    if (p.window == 8) {
        switch (nqp) {
            case 16: return launch_unit_t<16, 8>(p, n_units, smem, stream);
            case 32: return launch_unit_t<32, 8>(p, n_units, smem, stream);
            case 48: return launch_unit_t<48, 8>(p, n_units, smem, stream);
            case 64: return launch_unit_t<64, 8>(p, n_units, smem, stream);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (nqp) {
        case 16: return launch_unit_t<16, 0>(p, n_units, smem, stream);
        case 32: return launch_unit_t<32, 0>(p, n_units, smem, stream);
        case 48: return launch_unit_t<48, 0>(p, n_units, smem, stream);
        case 64: return launch_unit_t<64, 0>(p, n_units, smem, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace rkv
