// pgd_decode.cuh -- split-KV paged GQA decode attention kernel for sm_100a.
//
// What it computes ("attention kernels", froggydisk: sections "standard
// attention", "FlashAttention", "prefill and decode attention", "paged KV and
// kernels"; "batching and attention", beengineer500, sections 2.4 and 3.4):
// for every sequence s and query head i (KV head h = i / g)
//     out[s][i] = softmax(scale * q[s][i] . K_t) . V_t  over t < context_lens[s],
// with K_t / V_t read through the block table, and lse[s][i] its log-sum-exp.
//
// Work decomposition.  The batch is flattened into tiles (s, h, j): KV head h
// of logical block j of sequence s, ordered by s, then h, then j.  The U tiles
// are cut into gridDim.x equal contiguous ranges, one per CTA, so every CTA
// streams the same number of KV bytes whatever the length mix ("prefill and
// decode attention": split along the KV length so all SMs read at once).
// Every CTA derives the cut from context_lens itself (no host round trip).
// Inside its range a CTA walks "segments" (the part of one (s, h) unit that
// falls in the range).  A segment that covers its whole unit writes `out`
// directly; otherwise it writes a partial (o, lse) and the CTA that completes
// the unit's last share merges the partials by log-sum-exp.
//
// CTA = 4 consumer warps + 1 producer warp.  The producer walks the same
// segments and issues one TMA tensor load per (block, KV head) tile of K and
// of V into a ring of shared-memory stages (64 tokens each, 128-byte swizzle,
// mbarrier completion).  Each K/V tile is fetched once and used by all g
// query heads of the group ("prefill and decode attention": GQA reuse).
//
// Per stage the consumers run a small tensor-core contraction per warp
// (mma.sync m16n8k16, fp32 accumulate) with the roles transposed so that the
// group's query heads are the narrow N = 8 dimension:
//   S^T[tokens][heads] = K[tokens][d] . Q^T[d][heads]   (each warp: 16 tokens)
//   stage max per head through shared memory -> p = exp2(S - m)
//   O^T[d][heads] += V^T[d][tokens] . P^T[tokens][heads] (each warp: D/4 dims)
// which is the online softmax of "FlashAttention" applied stage by stage.
// With bf16 K/V the weights p enter the PV product as two bf16 terms,
// p_hi = bf16(p) and p_lo = bf16(p - p_hi) (about 16 significant bits), and
// the normaliser sums the fp32 p; with FP8 K/V they enter as f16 (11 bits)
// and the normaliser sums those rounded values.
#pragma once

#include "pgd_ptx.cuh"

namespace pgd {

struct DecodeParams {
    const uint16_t *q;            // bf16 bits [B][Hq][D]
    uint16_t *out;                // bf16 bits [B][Hq][D]
    float *lse_out;               // [B][Hq] natural log, may be null
    const int32_t *block_table;   // [B][max_blocks_per_seq]
    const int32_t *context_lens;  // [B]
    const float *k_scale;         // [Hkv] (FP8 only)
    const float *v_scale;
    int32_t *counters;            // [B * Hkv], zero between calls (library-owned)
    float *o_part;                // [2 * grid][g][D]
    float *lse_part;              // [2 * grid][g], log2 domain
    uint32_t *flags;              // device flag word
    int32_t max_blocks_per_seq;
    int32_t num_seqs, num_q_heads, num_kv_heads, group, num_blocks;
    float scale_log2;             // softmax scale * log2(e)
};

constexpr int kConsumerWarps = 4;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kStageTokens = 16 * kConsumerWarps;
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kBarConsumers = 1;

template <int D, int BS, int NT, bool FP8, int NSTAGES>
struct DecodeCfg {
    static constexpr int E = FP8 ? 1 : 2;                // bytes per KV element
    static constexpr int ROW = D * E;                    // bytes per K/V row
    static constexpr int LINES = ROW / 128;              // 128-byte lines per row
    static constexpr int TILE = BS * ROW;                // one (block, head) tile
    static constexpr int BPS = kStageTokens / BS;        // blocks per stage
    static constexpr int STAGE_KV = BPS * TILE;          // K (or V) bytes per stage
    static constexpr int STAGE = 2 * STAGE_KV;
    static constexpr int NP = 8 * NT;                    // padded heads per unit
    static constexpr int DW = D / kConsumerWarps;        // PV dims per warp
    static constexpr int MT = DW / 16;                   // PV m-tiles per warp
    static constexpr int KSTEPS = D / 16;                // QK k-steps
    // shared memory carve-up (offsets from a 1024-aligned base)
    static constexpr int OFF_P = NSTAGES * STAGE;
    static constexpr int P_BYTES = kStageTokens * NP * 2;   // one weight plane
    static constexpr int OFF_RED = OFF_P + 2 * P_BYTES;      // hi and lo planes
    static constexpr int OFF_LSUM = OFF_RED + kConsumerWarps * NP * 4;
    static constexpr int OFF_BAR = OFF_LSUM + kConsumerWarps * NP * 4;
    static constexpr int OFF_MISC = OFF_BAR + 2 * NSTAGES * 8;
    static constexpr int MISC_BYTES = 256;
    static constexpr int SMEM = OFF_MISC + MISC_BYTES + 1024;   // + alignment slack
    static_assert(ROW % 128 == 0, "rows must be whole 128-byte lines");
    static_assert(kStageTokens % BS == 0, "stage must hold whole blocks");
    static_assert(!FP8 || D == 128, "FP8 path is compiled for head_dim 128");
    static_assert(TILE % 1024 == 0, "tiles must keep the 1024-byte swizzle atom aligned");
};

struct Misc {                 // CTA-wide scalars in shared memory
    long long u0, u1, total;  // tile range of this CTA, total tiles
    long long pfx0;           // flattened index of the first tile of unit (s0, *)
    int s0;
    int is_last;
    int found;
    long long warp_tmp[8];
};

// ------------------------------------------------------------------ helpers
template <int BS>
__device__ __forceinline__ int ctx_of(const DecodeParams &p, int s) {
    int n = __ldg(p.context_lens + s);
    const int cap = p.max_blocks_per_seq * BS;
    if (n < 0 || n > cap) {
        raise_flag(p.flags, kFlagContextLen);
        n = n < 0 ? 0 : cap;
    }
    return n;
}

template <int BS>
__device__ __forceinline__ int nblk_of(int ctx) { return (ctx + BS - 1) / BS; }

// Block-wide sum over all kThreads threads (int64).
__device__ __forceinline__ long long block_sum(long long v, Misc *m) {
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) m->warp_tmp[w] = v;
    __syncthreads();
    long long t = 0;
    for (int i = 0; i < kThreads / 32; ++i) t += m->warp_tmp[i];
    __syncthreads();
    return t;
}

// Block-wide inclusive scan over kThreads threads (int64); also returns the
// block total.
__device__ __forceinline__ long long block_scan(long long v, long long &total, Misc *m) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int o = 1; o < 32; o <<= 1) {
        long long n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    __syncthreads();
    if (lane == 31) m->warp_tmp[w] = v;
    __syncthreads();
    long long before = 0;
    total = 0;
    for (int i = 0; i < kThreads / 32; ++i) {
        if (i < w) before += m->warp_tmp[i];
        total += m->warp_tmp[i];
    }
    __syncthreads();
    return v + before;
}

// First CTA whose range contains flattened tile x (ranges are
// [c*U/G, (c+1)*U/G)).
__device__ __forceinline__ long long cta_of(long long x, long long U, long long G) {
    return ((x + 1) * G - 1) / U;
}

// Walk state shared by producer and consumers (same deterministic order).
struct Cursor {
    int s, h, j, n, ctx;
    long long u;
};

template <int BS>
__device__ __forceinline__ void next_unit(Cursor &c, const DecodeParams &p) {
    c.j = 0;
    if (++c.h == p.num_kv_heads) {
        c.h = 0;
        for (++c.s; c.s < p.num_seqs; ++c.s) {
            c.ctx = ctx_of<BS>(p, c.s);
            c.n = nblk_of<BS>(c.ctx);
            if (c.n) break;
        }
    }
}

// ------------------------------------------------------------------ kernel
template <int D, int BS, int NT, bool FP8, int NSTAGES>
__global__ void __launch_bounds__(kThreads)
paged_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
    using C = DecodeCfg<D, BS, NT, FP8, NSTAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    Misc *misc = reinterpret_cast<Misc *>(smem + C::OFF_MISC);
    float *red = reinterpret_cast<float *>(smem + C::OFF_RED);
    float *lsum = reinterpret_cast<float *>(smem + C::OFF_LSUM);
    const uint32_t bar_full = sbase + C::OFF_BAR;
    const uint32_t bar_empty = bar_full + NSTAGES * 8;
    const uint32_t sP = sbase + C::OFF_P;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.num_seqs, Hkv = p.num_kv_heads, g = p.group;
    const long long cta = blockIdx.x;

    if (tid == 0) {
        for (int i = 0; i < NSTAGES; ++i) {
            mbar_init(bar_full + 8 * i, 1);
            mbar_init(bar_empty + 8 * i, kConsumerWarps);
        }
        fence_mbar_init();
        misc->found = 0;
    }
    if (warp == kConsumerWarps && lane == 0) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }

    // ---- prologue: total tiles and this CTA's range --------------------
    long long mine = 0;
    for (int s = tid; s < B; s += kThreads) mine += nblk_of<BS>(ctx_of<BS>(p, s));
    const long long U = block_sum(mine, misc) * Hkv;
    // CTAs beyond the tile count get no range, so every range is non-empty
    const long long G = min((long long)gridDim.x, U);
    const long long u0 = cta < G ? cta * U / G : 0, u1 = cta < G ? (cta + 1) * U / G : 0;

    // units with an empty context: out = 0, lse = -inf (spread over CTAs)
    for (long long v = cta; v < (long long)B * Hkv; v += gridDim.x) {
        const int s = (int)(v / Hkv), h = (int)(v % Hkv);
        if (ctx_of<BS>(p, s) != 0) continue;
        uint16_t *o = p.out + ((long long)s * p.num_q_heads + (long long)h * g) * D;
        for (int e = tid; e < g * D; e += kThreads) o[e] = 0;
        if (p.lse_out && tid < g) p.lse_out[(long long)s * p.num_q_heads + h * g + tid] = -INFINITY;
    }
    if (u0 >= u1) return;   // nothing in flight, no barrier shared past this point

    // locate the unit that holds tile u0
    {
        long long base = 0;
        for (int sb = 0; sb < B; sb += kThreads) {
            const int s = sb + tid;
            const long long wgt = s < B ? (long long)nblk_of<BS>(ctx_of<BS>(p, s)) * Hkv : 0;
            long long tot;
            const long long incl = block_scan(wgt, tot, misc);
            const long long excl = base + incl - wgt;
            if (s < B && wgt > 0 && excl <= u0 && u0 < excl + wgt) {
                misc->s0 = s;
                misc->pfx0 = excl;
                misc->found = 1;
            }
            base += tot;
            __syncthreads();
            if (misc->found) break;
        }
    }
    __syncthreads();

    Cursor cur;
    cur.s = misc->s0;
    cur.ctx = ctx_of<BS>(p, cur.s);
    cur.n = nblk_of<BS>(cur.ctx);
    {
        const long long off = u0 - misc->pfx0;
        cur.h = (int)(off / cur.n);
        cur.j = (int)(off % cur.n);
    }
    cur.u = u0;

    if (warp == kConsumerWarps) {
        // ================= producer: one lane issues all TMA loads ========
        if (lane != 0) return;
        uint32_t it = 0;
        bool ok = true;
        while (cur.u < u1 && ok) {
            const int j1 = (int)min((long long)cur.n, cur.j + (u1 - cur.u));
            const int32_t *bt = p.block_table + (long long)cur.s * p.max_blocks_per_seq;
            for (int jj = cur.j; jj < j1 && ok; jj += C::BPS) {
                const int nb = min(C::BPS, j1 - jj);
                const uint32_t slot = it % NSTAGES;
                if (it >= NSTAGES) {
                    ok = mbar_wait_bounded(bar_empty + 8 * slot, ((it / NSTAGES) - 1) & 1);
                    if (!ok) { raise_flag(p.flags, kFlagTimeout); break; }
                }
                const uint32_t full = bar_full + 8 * slot;
                mbar_arrive_expect_tx(full, (uint32_t)(nb * 2 * C::TILE));
                const uint32_t dK = sbase + slot * C::STAGE, dV = dK + C::STAGE_KV;
                for (int b = 0; b < nb; ++b) {
                    int pb = __ldg(bt + jj + b);
                    if (pb < 0 || pb >= p.num_blocks) {
                        raise_flag(p.flags, kFlagBlockId);
                        pb = 0;
                    }
                    const int32_t row = pb * Hkv + cur.h;
                    tma_load_4d(dK + b * C::TILE, &tmK, full, 0, 0, 0, row);
                    tma_load_4d(dV + b * C::TILE, &tmV, full, 0, 0, 0, row);
                }
                ++it;
            }
            cur.u += j1 - cur.j;
            next_unit<BS>(cur, p);
        }
        // drain: every issued stage must land before the CTA may exit
        const uint32_t first = it > NSTAGES ? it - NSTAGES : 0;
        for (uint32_t k = first; k < it; ++k)
            if (!mbar_wait_bounded(bar_full + 8 * (k % NSTAGES), (k / NSTAGES) & 1, 200000000ull))
                raise_flag(p.flags, kFlagTimeout);
        return;
    }

    // ==================== consumers (warps 0..3) ===========================
    const int gid = lane >> 2, t4 = lane & 3;
    uint32_t it = 0;

    while (cur.u < u1) {
        const int j0 = cur.j;
        const int j1 = (int)min((long long)cur.n, cur.j + (u1 - cur.u));
        const int s = cur.s, h = cur.h, ctx = cur.ctx;
        const bool whole = (j0 == 0 && j1 == cur.n);

        // ---- query fragments (B operand, Q^T[d][head]) for this unit ----
        uint32_t qf[C::KSTEPS][NT][2];
        {
            const uint16_t *qb = p.q + ((long long)s * p.num_q_heads + (long long)h * g) * D;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int head = nt * 8 + gid;
                const bool live = head < g;
                const uint32_t *qr = reinterpret_cast<const uint32_t *>(qb + (live ? head : 0) * D);
#pragma unroll
                for (int k = 0; k < C::KSTEPS; ++k) {
                    uint32_t b0, b1;
                    if (!FP8) {   // k index 2t, 2t+1 | 2t+8, 2t+9  <->  same d
                        b0 = __ldg(qr + (16 * k + 2 * t4) / 2);
                        b1 = __ldg(qr + (16 * k + 8 + 2 * t4) / 2);
                    } else {      // k index permuted to d = 16k + 4t + {0,1 | 2,3}
                        b0 = bf16x2_to_f16x2(__ldg(qr + (16 * k + 4 * t4) / 2));
                        b1 = bf16x2_to_f16x2(__ldg(qr + (16 * k + 4 * t4 + 2) / 2));
                    }
                    qf[k][nt][0] = live ? b0 : 0u;
                    qf[k][nt][1] = live ? b1 : 0u;
                }
            }
        }
        float sl2 = p.scale_log2, vsc = 1.f;
        if (FP8) {
            sl2 *= __ldg(p.k_scale + h);
            vsc = __ldg(p.v_scale + h);
        }

        float m_run[NT][2], l_run[NT][2];
        float o_acc[C::MT][NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            m_run[nt][0] = m_run[nt][1] = -INFINITY;
            l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
            for (int mt = 0; mt < C::MT; ++mt)
                o_acc[mt][nt][0] = o_acc[mt][nt][1] = o_acc[mt][nt][2] = o_acc[mt][nt][3] = 0.f;
        }

        for (int jj = j0; jj < j1; jj += C::BPS) {
            const int nb = min(C::BPS, j1 - jj);
            const int n_valid = min(ctx - jj * BS, nb * BS);
            const uint32_t slot = it % NSTAGES;
            const bool ok = mbar_wait_bounded(bar_full + 8 * slot, (it / NSTAGES) & 1);
            if (!ok) raise_flag(p.flags, kFlagTimeout);
            const uint32_t sK = sbase + slot * C::STAGE, sV = sK + C::STAGE_KV;

            // ---- S^T = K . Q^T for this warp's 16 tokens ----------------
            float sacc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
            if (16 * warp < n_valid) {
                if (!FP8) {
                    const int mi = lane >> 3;
                    const int tok = 16 * warp + (mi & 1) * 8 + (lane & 7);
                    const int row = tok % BS;
                    const uint32_t rowaddr = sK + (tok / BS) * C::TILE + row * 128;
#pragma unroll
                    for (int k = 0; k < C::KSTEPS; ++k) {
                        const int chunk = 2 * k + (mi >> 1);
                        const uint32_t addr = rowaddr + (chunk >> 3) * (BS * 128) +
                                              (((chunk & 7) ^ (row & 7)) << 4);
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4(addr, a0, a1, a2, a3);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            mma_bf16(sacc[nt], a0, a1, a2, a3, qf[k][nt][0], qf[k][nt][1]);
                    }
                } else {
                    const int tok0 = 16 * warp + gid, tok1 = tok0 + 8;
                    const int r0 = tok0 % BS, r1 = tok1 % BS;
                    const uint32_t base0 = sK + (tok0 / BS) * C::TILE + r0 * 128 + 4 * t4;
                    const uint32_t base1 = sK + (tok1 / BS) * C::TILE + r1 * 128 + 4 * t4;
#pragma unroll
                    for (int k = 0; k < C::KSTEPS; ++k) {
                        uint32_t w0, w1;
                        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(w0) : "r"(base0 + ((k ^ (r0 & 7)) << 4)));
                        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(w1) : "r"(base1 + ((k ^ (r1 & 7)) << 4)));
                        const uint32_t a0 = e4m3x2_to_f16x2(w0 & 0xffffu);
                        const uint32_t a2 = e4m3x2_to_f16x2(w0 >> 16);
                        const uint32_t a1 = e4m3x2_to_f16x2(w1 & 0xffffu);
                        const uint32_t a3 = e4m3x2_to_f16x2(w1 >> 16);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            mma_f16(sacc[nt], a0, a1, a2, a3, qf[k][nt][0], qf[k][nt][1]);
                    }
                }
            }

            // ---- scale, mask, stage max per head -------------------------
            float mx[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tok = 16 * warp + gid + (e >> 1) * 8;
                    const int head = nt * 8 + 2 * t4 + (e & 1);
                    sacc[nt][e] = (tok < n_valid && head < g) ? sacc[nt][e] * sl2 : -INFINITY;
                }
                mx[nt][0] = fmaxf(sacc[nt][0], sacc[nt][2]);
                mx[nt][1] = fmaxf(sacc[nt][1], sacc[nt][3]);
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) {
                    mx[nt][0] = fmaxf(mx[nt][0], __shfl_xor_sync(0xffffffffu, mx[nt][0], o));
                    mx[nt][1] = fmaxf(mx[nt][1], __shfl_xor_sync(0xffffffffu, mx[nt][1], o));
                }
                if (gid == 0) {
                    red[warp * C::NP + nt * 8 + 2 * t4] = mx[nt][0];
                    red[warp * C::NP + nt * 8 + 2 * t4 + 1] = mx[nt][1];
                }
            }
            named_bar_sync(kBarConsumers, kConsumers);

            // ---- new running max, probabilities to shared memory -----------
            float alpha[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float sm = red[nt * 8 + 2 * t4 + e];
#pragma unroll
                    for (int w = 1; w < kConsumerWarps; ++w)
                        sm = fmaxf(sm, red[w * C::NP + nt * 8 + 2 * t4 + e]);
                    const float m_new = fmaxf(m_run[nt][e], sm);
                    const float m_use = m_new == -INFINITY ? 0.f : m_new;
                    alpha[nt][e] = ex2(m_run[nt][e] - m_use);
                    m_run[nt][e] = m_new;
                    mx[nt][e] = m_use;
                }
                float pr[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) pr[e] = ex2(sacc[nt][e] - mx[nt][e & 1]);
                const int tok = 16 * warp + gid;
                const uint32_t pa = sP + (tok * C::NP + nt * 8 + 2 * t4) * 2;
                const uint32_t row8 = 8 * C::NP * 2;          // token + 8
                if (!FP8) {
                    // p = hi + lo, both bf16; the normaliser sums the fp32 p
                    const uint32_t h0 = pack_bf16x2(pr[0], pr[1]);
                    const uint32_t h1 = pack_bf16x2(pr[2], pr[3]);
                    const float2 r0 = unpack_bf16x2(h0), r1 = unpack_bf16x2(h1);
                    const uint32_t l0 = pack_bf16x2(pr[0] - r0.x, pr[1] - r0.y);
                    const uint32_t l1 = pack_bf16x2(pr[2] - r1.x, pr[3] - r1.y);
                    l_run[nt][0] = l_run[nt][0] * alpha[nt][0] + pr[0] + pr[2];
                    l_run[nt][1] = l_run[nt][1] * alpha[nt][1] + pr[1] + pr[3];
                    asm volatile("st.shared.b32 [%0], %1;" ::"r"(pa), "r"(h0));
                    asm volatile("st.shared.b32 [%0], %1;" ::"r"(pa + row8), "r"(h1));
                    asm volatile("st.shared.b32 [%0], %1;" ::"r"(pa + C::P_BYTES), "r"(l0));
                    asm volatile("st.shared.b32 [%0], %1;" ::"r"(pa + C::P_BYTES + row8), "r"(l1));
                } else {
                    // f16 weights; the normaliser sums exactly the rounded values
                    const uint32_t h0 = pack_f16x2(pr[0], pr[1]);
                    const uint32_t h1 = pack_f16x2(pr[2], pr[3]);
                    const float2 r0 = unpack_f16x2(h0), r1 = unpack_f16x2(h1);
                    l_run[nt][0] = l_run[nt][0] * alpha[nt][0] + r0.x + r1.x;
                    l_run[nt][1] = l_run[nt][1] * alpha[nt][1] + r0.y + r1.y;
                    asm volatile("st.shared.b32 [%0], %1;" ::"r"(pa), "r"(h0));
                    asm volatile("st.shared.b32 [%0], %1;" ::"r"(pa + row8), "r"(h1));
                }
            }
            // rows past the end of the context may hold anything (NaN, Inf):
            // zero this warp's invalid V rows so that 0 * V stays 0.
            if (n_valid < kStageTokens) {
                const int first = max(16 * warp, n_valid), last = 16 * warp + 16;
                const int lines = (last - first) * C::LINES;
                for (int i = lane >> 3; i < lines; i += 4) {
                    const int tok = first + i / C::LINES, ln = i % C::LINES;
                    const uint32_t a = sV + (tok / BS) * C::TILE + ln * (BS * 128) +
                                       (tok % BS) * 128 + (lane & 7) * 16;
                    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0));
                }
                // order these generic-proxy writes before the next TMA into the slot
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            }
            // all consumers agree on whether any of them timed out
            const bool abort = named_bar_sync_or(kBarConsumers, kConsumers, !ok);

            // ---- O^T += V^T . P^T for this warp's D/4 dims ------------------
#pragma unroll
            for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    o_acc[mt][nt][0] *= alpha[nt][0];
                    o_acc[mt][nt][1] *= alpha[nt][1];
                    o_acc[mt][nt][2] *= alpha[nt][0];
                    o_acc[mt][nt][3] *= alpha[nt][1];
                }
#pragma unroll
            for (int kk = 0; kk < kStageTokens / 16; ++kk) {
                if (16 * kk >= n_valid) break;
                uint32_t pb[NT][2], pl[NT][2];
                {
                    const int mi = lane >> 3;
                    const int tok = 16 * kk + 8 * (mi & 1) + (lane & 7);
                    const uint32_t pa = NT == 1 ? sP + tok * C::NP * 2
                                                : sP + (tok * C::NP + 8 * (mi >> 1)) * 2;
                    if (NT == 1) {
                        ldsm_x2_t(pa, pb[0][0], pb[0][1]);
                        if (!FP8) ldsm_x2_t(pa + C::P_BYTES, pl[0][0], pl[0][1]);
                    } else {
                        ldsm_x4_t(pa, pb[0][0], pb[0][1], pb[NT - 1][0], pb[NT - 1][1]);
                        if (!FP8)
                            ldsm_x4_t(pa + C::P_BYTES, pl[0][0], pl[0][1], pl[NT - 1][0],
                                      pl[NT - 1][1]);
                    }
                }
                if (!FP8) {
                    const int mi = lane >> 3;
                    const int tok = 16 * kk + (mi >> 1) * 8 + (lane & 7);
                    const int row = tok % BS;
                    const uint32_t rowaddr = sV + (tok / BS) * C::TILE + row * 128;
#pragma unroll
                    for (int mt = 0; mt < C::MT; ++mt) {
                        const int chunk = (C::DW * warp + 16 * mt) / 8 + (mi & 1);
                        const uint32_t addr = rowaddr + (chunk >> 3) * (BS * 128) +
                                              (((chunk & 7) ^ (row & 7)) << 4);
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4_t(addr, a0, a1, a2, a3);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            mma_bf16(o_acc[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
                            mma_bf16(o_acc[mt][nt], a0, a1, a2, a3, pl[nt][0], pl[nt][1]);
                        }
                    }
                } else {
                    // rows 2t, 2t+1, 2t+8, 2t+9 of this k-step; 4 bytes at
                    // d = 32*warp + 4*gid (m-tile 0: +0,+1; m-tile 1: +2,+3)
                    const int chunk = 2 * warp + (gid >> 2);
                    uint32_t wv[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int tok = 16 * kk + 2 * t4 + (q & 1) + (q >> 1) * 8;
                        const int row = tok % BS;
                        const uint32_t a = sV + (tok / BS) * C::TILE + row * 128 +
                                           ((chunk ^ (row & 7)) << 4) + 4 * (gid & 3);
                        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(wv[q]) : "r"(a));
                    }
#pragma unroll
                    for (int mt = 0; mt < C::MT; ++mt) {
                        const uint32_t sel = mt == 0 ? 0x5140u : 0x7362u;
                        const uint32_t x = prmt(wv[0], wv[1], sel);
                        const uint32_t y = prmt(wv[2], wv[3], sel);
                        const uint32_t a0 = e4m3x2_to_f16x2(x & 0xffffu);
                        const uint32_t a1 = e4m3x2_to_f16x2(x >> 16);
                        const uint32_t a2 = e4m3x2_to_f16x2(y & 0xffffu);
                        const uint32_t a3 = e4m3x2_to_f16x2(y >> 16);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
                            mma_f16(o_acc[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_empty + 8 * slot);
            ++it;
            if (abort) return;   // uniform over the consumers; the producer drains
        }

        // ---- finish the segment ---------------------------------------------
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float v = l_run[nt][e];
                for (int o = 4; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (gid == 0) lsum[warp * C::NP + nt * 8 + 2 * t4 + e] = v;
            }
        named_bar_sync(kBarConsumers, kConsumers);
        float inv_l[NT][2], lse2[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float l = 0.f;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) l += lsum[w * C::NP + nt * 8 + 2 * t4 + e];
                inv_l[nt][e] = l > 0.f ? vsc / l : 0.f;
                lse2[nt][e] = l > 0.f ? m_run[nt][e] + log2f(l) : -INFINITY;
            }

        // output dim held by accumulator element (mt, e)
        auto dim_of = [&](int mt, int e) -> int {
            if (!FP8) return C::DW * warp + 16 * mt + gid + (e >> 1) * 8;
            return 32 * warp + 4 * gid + 2 * mt + (e >> 1);
        };
        const long long row0 = (long long)s * p.num_q_heads + (long long)h * g;
        if (whole) {
#pragma unroll
            for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int head = nt * 8 + 2 * t4 + (e & 1);
                        if (head < g) {
                            const float v = o_acc[mt][nt][e] * inv_l[nt][e & 1];
                            p.out[(row0 + head) * D + dim_of(mt, e)] =
                                __bfloat16_as_ushort(__float2bfloat16_rn(v));
                        }
                    }
            if (p.lse_out && warp == 0 && gid == 0) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int head = nt * 8 + 2 * t4 + e;
                        if (head < g) p.lse_out[row0 + head] = lse2[nt][e] * kLn2;
                    }
            }
        } else {
            // partial: slot 2c for the CTA's first segment, 2c+1 for its last
            const bool first_seg = (cur.u == u0);
            const long long slot = 2 * cta + (first_seg ? 0 : 1);
            float *op = p.o_part + slot * g * D;
#pragma unroll
            for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int head = nt * 8 + 2 * t4 + (e & 1);
                        if (head < g) op[head * D + dim_of(mt, e)] = o_acc[mt][nt][e] * inv_l[nt][e & 1];
                    }
            if (warp == 0 && gid == 0) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int head = nt * 8 + 2 * t4 + e;
                        if (head < g) p.lse_part[slot * g + head] = lse2[nt][e];
                    }
            }
            __threadfence();
            named_bar_sync(kBarConsumers, kConsumers);
            // unit tile range [ua, ub) and the CTAs that share it
            const long long ua = cur.u - j0;   // flattened index of tile (s, h, 0)
            const long long ub = ua + cur.n;
            const long long c_first = cta_of(ua, U, G), c_last = cta_of(ub - 1, U, G);
            if (tid == 0) {
                const int prev = atomicAdd(p.counters + (long long)s * Hkv + h, 1);
                misc->is_last = (prev == (int)(c_last - c_first));
            }
            named_bar_sync(kBarConsumers, kConsumers);
            if (misc->is_last) {
                __threadfence();
                for (int e = tid; e < g * D; e += kConsumers) {
                    const int head = e / D, d = e % D;
                    float M = -INFINITY;
                    for (long long c = c_first; c <= c_last; ++c) {
                        const long long sl = 2 * c + ((ua <= c * U / G) ? 0 : 1);
                        M = fmaxf(M, __ldcg(p.lse_part + sl * g + head));
                    }
                    const float Mu = M == -INFINITY ? 0.f : M;
                    float W = 0.f, acc = 0.f;
                    for (long long c = c_first; c <= c_last; ++c) {
                        const long long sl = 2 * c + ((ua <= c * U / G) ? 0 : 1);
                        const float w = ex2(__ldcg(p.lse_part + sl * g + head) - Mu);
                        W += w;
                        acc += w * __ldcg(p.o_part + (sl * g + head) * D + d);
                    }
                    p.out[(row0 + head) * D + d] =
                        __bfloat16_as_ushort(__float2bfloat16_rn(W > 0.f ? acc / W : 0.f));
                    if (p.lse_out && d == 0)
                        p.lse_out[row0 + head] = W > 0.f ? (M + log2f(W)) * kLn2 : -INFINITY;
                }
                if (tid == 0) p.counters[(long long)s * Hkv + h] = 0;
            }
        }

        cur.u += j1 - j0;
        next_unit<BS>(cur, p);
    }
}

}  // namespace pgd
