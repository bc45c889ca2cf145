// rkv_gram.cu -- MAX-mode redundancy on the tensor cores:
//   r_i = max_{j < N, j != i} khat_i . khat_j,  khat = k / max(||k||, 1e-12),
// for every candidate i < M of every due unit.  Redundancy is the cosine
// similarity of key vectors ("R-KV: Redundancy-aware KV Cache Compression for
// Reasoning Models", atlas.scime.ai summary, "Approach"); the max over the
// other keys is the near-duplicate reading of "cosine similarity to identify
// and prune near-duplicates" (sourcepulse summary, "How It Works").
//
// With a_ij = k_i . k_j (bf16 products, fp32 accumulate on tcgen05) and
// inv_i = 1 / max(||k_i||, 1e-12):  r_i = inv_i * u_i,  u_i = max_{j != i} a_ij inv_j.
// The Gram matrix is symmetric, so only the tile pairs (I <= J) of 128 x 128 are
// computed: the accumulator of pair (I, J) gives u of the rows of tile I (row
// maxima of a_ij inv_j) and of the rows of tile J (column maxima of a_ij inv_i).
// The N x N matrix never leaves the chip, and the inverse norms come from its
// diagonal (||k_j||^2 = a_jj of the diagonal pair (J, J)): K is read once from
// HBM (the tiles a unit reuses come from L2).
//
// Persistent CTAs (one per SM) walk the units.  Per unit the column tiles J go
// from first to last; tile J stays resident while the row tiles I = J (the
// diagonal, from the resident tile itself), 0, 1, ..., J-1 stream past it, so
// every row tile's inverse norms are known when it arrives, and the column
// maxima of tile J build up in registers over the whole column and cross lanes
// once.  Warp roles (576 threads, one CTA per SM):
//   warps 0-15 epilogue, warp w on TMEM lane quadrant w % 4 and column quarter
//              w / 4: per pair, the accumulator read with tcgen05.ld 16x256b
//              (each thread holds 4 rows x 8 columns); row maxima folded over
//              the 8 columns and across the 4 lanes of a row group, merged into
//              per-row order-preserving keys in shared memory with atomicMax;
//              column maxima kept per thread until the column tile is done,
//              then folded across the 8 lanes of a column group and merged the
//              same way.  On the diagonal pair of each column tile the four
//              warps with qd == cq turn its diagonal into the tile's inverse
//              norms, published to all epilogue warps by one named barrier;
//   warp 16    producer: TMA of the column tile (double-buffered) and of the
//              row tiles (three-stage ring);
//   warp 17    MMA issuer: 8 UMMAs (K = 128) per pair, issued from one asm
//              block, into one of four TMEM accumulators (128 columns each).
// Hand-offs are mbarriers; every wait is bounded and a timeout is recorded in
// the status word (the CTA then drains what it issued and stops).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "rkv_block.cuh"
#include "rkv_internal.h"
#include "rkv_ptx.cuh"

namespace rkv {

namespace {

constexpr int kEpiWarps = 16;                     // 4 TMEM quadrants x 4 column quarters
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kGramThreads = kEpiThreads + 64;     // + producer warp + MMA warp
constexpr int kProducerWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1;
constexpr int kBStages = 3;
constexpr int kAcc = 4;                            // TMEM accumulators of 128 columns
constexpr uint32_t kTileBytes = 128u * 256u;       // 128 rows x 128 bf16
constexpr uint32_t kHalfBytes = kTileBytes / 2;
constexpr uint32_t kTmemCols = 128u * kAcc;
constexpr uint32_t kBackoffNs = 64;              // producer / MMA polling interval

struct GramLayout {
    uint32_t a, b, key, inv, pages, bars, total;
};

// Offsets from a 1024-byte-aligned base; key and inv hold one entry per row of
// the largest unit (rounded up to whole tiles).
__host__ __device__ inline GramLayout gram_layout(int cap) {
    GramLayout L;
    const uint32_t kc = static_cast<uint32_t>((cap + 127) / 128) * 128u;
    uint32_t o = 0;
    L.a = o;     o += 2u * kTileBytes;
    L.b = o;     o += kBStages * kTileBytes;
    L.key = o;   o += 4u * kc;
    L.inv = o;   o += 4u * kc;
    L.pages = o; o += 4u * kUnitMaxPages;
    L.bars = o;  o += 256u;
    L.total = o + 1024u;
    return L;
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Order-preserving unsigned key of a float (larger float, larger key); 0 is
// below every key of a float, so a cleared array means "no value yet".
__device__ __forceinline__ uint32_t ord_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t k) {
    if (k == 0u) return -INFINITY;
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory"); }

// 16 TMEM lanes x 32 fp32 columns (16x256b, 4 repetitions): thread t gets, for
// repetition k, lane (t / 4) columns 8k + 2 (t % 4) + {0, 1} in r[4k], r[4k+1]
// and lane (t / 4) + 8 the same columns in r[4k+2], r[4k+3].
__device__ __forceinline__ void tmem_ld_16x256b_x4(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// The unit a persistent CTA handles k-th, its cache length and its rows.
struct UnitInfo {
    int N, M, T, b, h, l;
    int64_t unit_g, krow0;
};

__device__ __forceinline__ UnitInfo unit_info(const GramParams &p, int unit, int n_units) {
    UnitInfo u;
    const UnitCoord c = unit_coord(unit, p.n_kv, p.batch, n_units / (p.n_kv * p.batch), p.order);
    u.h = c.h;
    u.b = c.b;
    u.l = c.l;
    u.N = p.n_tokens_fixed > 0 ? p.n_tokens_fixed : p.n_eff[u.b];
    u.M = u.N - p.window;
    u.T = (u.N + 127) / 128;
    u.unit_g = (static_cast<int64_t>(p.layer_base + u.l) * p.batch + u.b) * p.n_kv + u.h;
    u.krow0 = unit_first_row(p.seq_row, p.seq_cap, u.b, u.h, p.n_kv, p.cap);
    return u;
}

}  // namespace

__global__ void __launch_bounds__(kGramThreads, 1) rkv_gram_max_kernel(const __grid_constant__ GramParams p,
                                                                      int n_units) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const GramLayout Lg = gram_layout(p.cap);
    uint8_t *sA = base + Lg.a;
    uint8_t *sB = base + Lg.b;
    uint32_t *sKey = reinterpret_cast<uint32_t *>(base + Lg.key);
    float *sInv = reinterpret_cast<float *>(base + Lg.inv);
    int32_t *sPages = reinterpret_cast<int32_t *>(base + Lg.pages);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + Lg.bars);
    uint64_t *afull = bars, *aempty = bars + 2, *bfull = bars + 4, *bempty = bars + 4 + kBStages;
    uint64_t *tfull = bars + 4 + 2 * kBStages, *tempty = tfull + kAcc;
    uint32_t *sTmem = reinterpret_cast<uint32_t *>(tempty + kAcc);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kc = (p.cap + 127) / 128 * 128;
    const bool paged = p.block_table != nullptr;
    const int psh = paged ? 31 - __clz(p.page_rows) : 7;
    const int P = 1 << psh;

    if (warp == 0) {
        tmem_alloc(sTmem, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 32) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&afull[i], 1);
            mbar_init(&aempty[i], 1);        // the column tile's last UMMA
        }
        for (int s = 0; s < kBStages; ++s) {
            mbar_init(&bfull[s], 1);
            mbar_init(&bempty[s], 1);
        }
        for (int t = 0; t < kAcc; ++t) {
            mbar_init(&tfull[t], 1);
            mbar_init(&tempty[t], kEpiWarps);   // one arrival per epilogue warp
        }
        fence_mbar_init();
    }
    for (int i = tid; i < kc; i += kGramThreads) sKey[i] = 0u;
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *sTmem;
    // a programmatic dependent of the plan kernel: nothing it wrote is read before this
    asm volatile("griddepcontrol.wait;" ::: "memory");

    bool ok = true;
    // buffers: sA = the resident column tiles (double-buffered), sB = the row-tile ring
    if (warp == kProducerWarp) {
        // ---------------- producer: per unit, column tiles 0 .. T-1; row tiles 0 .. J-1 of each
        uint32_t na = 0, nb = 0;
        for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x) {
            const UnitInfo u = unit_info(p, unit, n_units);
            if (u.N <= 0 || u.M <= 0) continue;
            const CUtensorMap *map = &p.tmap[u.l];
            if (paged) {
                __syncwarp();
                for (int j = lane; j < (u.N + P - 1) / P; j += 32)
                    sPages[j] = p.block_table[static_cast<int64_t>(u.b) * p.max_blocks + j];
                __syncwarp();
            }
            const int npg = (u.N + P - 1) / P;
            auto load_tile = [&](uint8_t *dst, uint64_t *bar, int t) {
                if (!paged) {
                    const int32_t y = static_cast<int32_t>(u.krow0 + t * 128);
                    tma_load_2d(dst, map, bar, 0, y);
                    tma_load_2d(dst + kHalfBytes, map, bar, 64, y);
                } else {
                    // one box per page; pages past the sequence's last read as zeros
                    for (int j = 0; j < 128 / P; ++j) {
                        const int pg = t * (128 / P) + j;
                        const int32_t y = pg < npg
                                              ? static_cast<int32_t>(((static_cast<int64_t>(sPages[pg]) * p.n_kv + u.h) << psh))
                                              : -P;
                        tma_load_2d(dst + j * P * 128, map, bar, 0, y);
                        tma_load_2d(dst + kHalfBytes + j * P * 128, map, bar, 64, y);
                    }
                }
            };
            for (int J = 0; J < u.T && ok; ++J) {
                if (lane == 0) {
                    const uint32_t a = na & 1u;
                    if (na >= 2 && !mbar_wait_backoff(&aempty[a], ((na >> 1) - 1) & 1u, kBackoffNs)) ok = false;
                    if (ok) {
                        mbar_arrive_expect_tx(&afull[a], kTileBytes);
                        load_tile(sA + a * kTileBytes, &afull[a], J);
                    }
                    ++na;
                    for (int I = 0; I < J && ok; ++I) {
                        const uint32_t s = nb % kBStages;
                        if (nb >= kBStages && !mbar_wait_backoff(&bempty[s], ((nb / kBStages) - 1) & 1u, kBackoffNs)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&bfull[s], kTileBytes);
                        load_tile(sB + s * kTileBytes, &bfull[s], I);
                        ++nb;
                    }
                }
                ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
            }
        }
        if (!ok && lane == 0) {
            // drain (bounded): the copies still in flight land before shared memory goes
            for (uint32_t i = na >= 2 ? na - 2 : 0; i < na; ++i)
                (void)mbar_wait(&afull[i & 1u], (i >> 1) & 1u);
            for (uint32_t i = nb >= kBStages ? nb - kBStages : 0; i < nb; ++i)
                (void)mbar_wait(&bfull[i % kBStages], (i / kBStages) & 1u);
        }
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issuer: D[i][j] = K_I[i] . K_J[j]; A = the row tile, B = the column tile
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
            uint32_t na = 0, nb = 0, np = 0;
            for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x) {
                const UnitInfo u = unit_info(p, unit, n_units);
                if (u.N <= 0 || u.M <= 0) continue;
                for (int J = 0; J < u.T && ok; ++J) {
                    const uint32_t a = na & 1u;
                    if (!mbar_wait_backoff(&afull[a], (na >> 1) & 1u, kBackoffNs)) { ok = false; break; }
                    ++na;
                    const uint32_t col_lo = desc_lo_sw128(smem_u32(sA + a * kTileBytes));
                    // the diagonal pair first (both operands the resident tile), then I = 0 .. J-1
                    for (int step = 0; step <= J && ok; ++step) {
                        const bool diag = step == 0;
                        const uint32_t t = np % kAcc;
                        if (np >= kAcc && !mbar_wait_backoff(&tempty[t], ((np / kAcc) - 1) & 1u, kBackoffNs)) { ok = false; break; }
                        uint32_t row_lo = col_lo, s = 0;
                        if (!diag) {
                            s = nb % kBStages;
                            if (!mbar_wait_backoff(&bfull[s], (nb / kBStages) & 1u, kBackoffNs)) { ok = false; break; }
                            row_lo = desc_lo_sw128(smem_u32(sB + s * kTileBytes));
                        }
                        tc_fence_after();
                        umma_bf16_k128_sw128(tmem_base + t * 128u, row_lo, col_lo, idesc);
                        umma_commit(&tfull[t]);
                        ++np;
                        if (!diag) {
                            umma_commit(&bempty[s]);
                            ++nb;
                        }
                    }
                    if (ok) umma_commit(&aempty[a]);
                }
            }
            // drain (bounded): every UMMA issued so far completes before TMEM is freed
            if (!ok && np > 0) (void)mbar_wait(&tfull[(np - 1) % kAcc], ((np - 1) / kAcc) & 1u);
        }
    } else {
        // ---------------- epilogue warps 0-15: quadrant qd of TMEM lanes, column quarter cq
        const int qd = warp & 3, cq = warp >> 2;
        const int g = lane >> 2, q = lane & 3;
        // this thread's 4 accumulator rows 32 qd + g + 8 r (r = 0, 1: the first 16-lane
        // slab, r = 2, 3: the second) and the row it keeps after the 4-lane fold (r = q);
        // its 8 columns 32 cq + 8 k + 2 q + e (k = 0..3, e = 0, 1)
        auto row_of = [&](int r) { return 32 * qd + g + 8 * r; };
        const int myrow = row_of(q);
        // the diagonal of the 32 x 32 block of a warp with qd == cq: lane (g, q = g / 2)
        // holds a_jj of columns 32 cq + 8 r + g (r = 0..3) in register e = g % 2 of (r, k = r)
        const bool diag_lane = qd == cq && q == (g >> 1);
        // A wait that runs out makes `ok` false for the whole warp (so the warp's
        // .sync.aligned TMEM loads never diverge); a failed warp skips the work but keeps
        // every named barrier of the schedule, so the other epilogue warps never wait
        // on it at a barrier without a time limit.
        auto wait_all = [&](uint64_t *bar, uint32_t parity) {
            const bool w = ok && mbar_wait(bar, parity);
            ok = __all_sync(kFull, w) != 0;
        };
        uint32_t np = 0;
        for (int unit = blockIdx.x; unit < n_units; unit += gridDim.x) {
            const UnitInfo u = unit_info(p, unit, n_units);
            if (u.N <= 0 || u.M <= 0) continue;
            for (int J = 0; J < u.T; ++J) {
                const int c0 = J * 128 + 32 * cq + 2 * q;    // unit row of this thread's column (k, e) = (0, 0)
                const bool tail = (J + 1) * 128 > u.N;       // columns past N in this tile
                float inv_c[8];                              // inverse norms of this thread's columns
                float colrun[8];                             // max over the rows seen of a_ij inv_i
#pragma unroll
                for (int c = 0; c < 8; ++c) colrun[c] = -INFINITY;
                for (int step = 0; step <= J; ++step) {
                    const bool diag = step == 0;
                    const int I = diag ? J : step - 1;
                    const uint32_t t = np % kAcc;
                    wait_all(&tfull[t], (np / kAcc) & 1u);
                    ++np;
                    uint32_t v0[16], v1[16];   // slab 0 (rows 0, 1), slab 1 (rows 2, 3)
                    if (ok) {
                        tc_fence_after();
                        const uint32_t tcol = tmem_base + t * 128u + 32u * cq;
                        tmem_ld_16x256b_x4(tcol + ((32u * qd) << 16), v0);
                        tmem_ld_16x256b_x4(tcol + ((32u * qd + 16u) << 16), v1);
                        tmem_wait_ld();
                        reg_tie16(v0);
                        reg_tie16(v1);
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tempty[t]);   // the accumulator may be reused
                    }
                    // a(row r, column k, e): slab r >> 1, register 4k + 2 (r & 1) + e
                    auto av = [&](int r, int k, int e) -> float {
                        const uint32_t x = (r < 2) ? v0[4 * k + 2 * (r & 1) + e] : v1[4 * k + 2 * (r & 1) + e];
                        return __uint_as_float(x);
                    };
                    if (diag) {
                        // 1 / max(||k_j||, 1e-12) of the column tile's rows (0 past N), with
                        // ||k_j||^2 = a_jj read off the diagonal of the tile's own Gram block;
                        // the barrier publishes them to every epilogue warp (rows of a later
                        // row tile are read by other warps than the one that wrote them)
                        if (ok && diag_lane) {
#pragma unroll
                            for (int r = 0; r < 4; ++r) {
                                const float ss = (g & 1) ? av(r, r, 1) : av(r, r, 0);
                                const int j = J * 128 + 32 * cq + 8 * r + g;
                                sInv[j] = j < u.N ? 1.0f / fmaxf(sqrtf(ss), 1e-12f) : 0.f;
                            }
                        }
                        epi_sync();
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float2 iv = *reinterpret_cast<const float2 *>(&sInv[c0 + 8 * k]);
                            inv_c[2 * k] = iv.x;
                            inv_c[2 * k + 1] = iv.y;
                        }
                    }
                    if (!ok) continue;
                    // ---- rows of tile I: max over this tile's columns of a_ij inv_j
                    float rm[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        float x[8];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float2 pr = __fmul2_rn(make_float2(av(r, k, 0), av(r, k, 1)),
                                                         make_float2(inv_c[2 * k], inv_c[2 * k + 1]));
                            x[2 * k] = pr.x;
                            x[2 * k + 1] = pr.y;
                        }
                        if (diag || tail) {
                            const int ri = I * 128 + row_of(r);
#pragma unroll
                            for (int k = 0; k < 4; ++k)
#pragma unroll
                                for (int e = 0; e < 2; ++e) {
                                    const int cj = c0 + 8 * k + e;
                                    if (cj == ri || cj >= u.N) x[2 * k + e] = -INFINITY;
                                }
                        }
                        rm[r] = fmax3(fmax3(x[0], x[1], x[2]), fmax3(x[3], x[4], x[5]), fmaxf(x[6], x[7]));
                    }
                    {
                        // fold across the 4 lanes of a row group: lane q keeps row q
                        const bool up = (q & 2) != 0;
                        const float s0 = up ? rm[0] : rm[2], s1 = up ? rm[1] : rm[3];
                        float k0 = up ? rm[2] : rm[0], k1 = up ? rm[3] : rm[1];
                        k0 = fmaxf(k0, __shfl_xor_sync(kFull, s0, 2));
                        k1 = fmaxf(k1, __shfl_xor_sync(kFull, s1, 2));
                        const bool up1 = (q & 1) != 0;
                        const float s2 = up1 ? k0 : k1;
                        float kk = up1 ? k1 : k0;
                        kk = fmaxf(kk, __shfl_xor_sync(kFull, s2, 1));
                        atomicMax(&sKey[I * 128 + myrow], ord_key(kk));
                    }
                    if (!diag) {
                        // ---- rows of tile J (this tile's columns): max over tile I's rows of
                        // a_ij inv_i, kept per thread until the column tile is done
                        // (the packed products pair the two adjacent columns of one row, whose
                        // accumulator values sit in adjacent registers)
                        float2 inv_r2[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const float v = sInv[I * 128 + row_of(r)];
                            inv_r2[r] = make_float2(v, v);
                        }
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            float2 y[4];
#pragma unroll
                            for (int r = 0; r < 4; ++r)
                                y[r] = __fmul2_rn(make_float2(av(r, k, 0), av(r, k, 1)), inv_r2[r]);
                            colrun[2 * k] = fmax3(fmax3(colrun[2 * k], y[0].x, y[1].x), y[2].x, y[3].x);
                            colrun[2 * k + 1] = fmax3(fmax3(colrun[2 * k + 1], y[0].y, y[1].y), y[2].y, y[3].y);
                        }
                    }
                }
                if (ok && J > 0) {
                    // fold the column maxima across the 8 lanes of a column group: lane g keeps
                    // column (k, e) = (g >> 1, g & 1) of its 8
#pragma unroll
                    for (int lvl = 0; lvl < 3; ++lvl) {
                        const int half = 4 >> lvl;              // values kept after this round
                        const int bit = 4 >> lvl;               // lane bit (of g) exchanged
                        const bool upper = (g & bit) != 0;
#pragma unroll
                        for (int i = 0; i < half; ++i) {
                            const float send = upper ? colrun[i] : colrun[i + half];
                            const float keep = upper ? colrun[i + half] : colrun[i];
                            colrun[i] = fmaxf(keep, __shfl_xor_sync(kFull, send, bit * 4));
                        }
                    }
                    atomicMax(&sKey[c0 + 8 * (g >> 1) + (g & 1)], ord_key(colrun[0]));
                }
            }
            // every key of the unit is final: r = inv_i * u_i; then clear for the next unit
            epi_sync();
            float *ro = p.r_out + u.unit_g * p.cap;
            for (int i = tid; i < u.T * 128; i += kEpiThreads) {
                if (i < u.M) ro[i] = key_value(sKey[i]) * sInv[i];
                sKey[i] = 0u;
            }
            epi_sync();
        }
    }
    if (!ok) record_flag(p.status, kDevFlagTimeout);
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

size_t gram_smem_bytes(int cap) { return gram_layout(cap).total; }

int gram_max_rows() {
    // rows whose keys and inverse norms still fit next to the tiles
    int cap = kUnitMaxRows;
    while (cap > 128 && gram_layout(cap).total > 232448u) cap -= 128;
    return cap;
}

cudaError_t launch_gram_max(const GramParams &p, int n_units, cudaStream_t stream,
                            cudaEvent_t before_gram, cudaEvent_t after_gram) {
    const size_t smem = gram_smem_bytes(p.cap);
    static std::atomic<int> granted{0};
    cudaError_t e = ensure_smem_attr(rkv_gram_max_kernel, smem, granted);
    if (e != cudaSuccess) return e;
    static int n_sm = 0;
    if (n_sm == 0) {
        int dev = 0, v = 0;
        e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        n_sm = v;
    }
    // launched as a programmatic dependent of the kernel before it: the CTAs may be
    // scheduled while it finishes, and wait for it on the device
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_units < n_sm ? n_units : n_sm), 1, 1);
    cfg.blockDim = dim3(kGramThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (before_gram) e = cudaEventRecord(before_gram, stream);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, rkv_gram_max_kernel, p, n_units);
    if (e == cudaSuccess && after_gram) e = cudaEventRecord(after_gram, stream);
    return e;
}

}  // namespace rkv
