// Backward pass of the chunked KDA prefill (fp32 SIMT arithmetic, every dtype and head size).
//
// The pages discuss training ("22,580" §6.1: prefill is the training-time path) but print no
// backward pass; this is the reverse-mode derivative of the chunk algorithm of "22,580" §6.3
// with the per-channel cumulative decay of its §08/§9.1 -- the same algebra as the forward:
// per chunk of C tokens with chunk-start state S, decay products D[r][i][c] =
// prod_{i<s<=r} alpha_s[c], gamma_r = prod_{s<=r} alpha_s, kappa_i = prod_{s>i} alpha_s,
//
//   K[r][i] = sum_c k_rc k_ic D_ric  (i < r),   A = Diag(beta) K,   T = (I + A)^{-1},
//   P[r][i] = s sum_c q_rc k_ic D_ric  (i <= r),  r = v - (k gamma) S,  u = T Diag(beta) r,
//   o = (s q gamma) S + P u,          S' = Diag(gamma_last) S + (k kappa)^T u.
//
// Given dO and dS' (the gradient of the chunk-end state), in the order computed below:
//   du  = P^T dO + (k kappa) dS'             dr = Diag(beta) T^T du = dv
//   dP  = tril(dO u^T)                       dT' = tril(du r^T)        (T' = T Diag(beta))
//   d(s q gamma) = dO S^T,   d(k gamma) = -dr S^T,   d(k kappa) = u dS'^T,
//   d gamma_last = rowsum(dS' * S)
//   dbeta_i += sum_r dT'_ri T_ri,  dT = dT' Diag(beta),  dA = strict-lower(-T^T dT T^T),
//   dbeta_r += sum_i dA_ri K_ri,   dK = Diag(beta) dA,
//   and through D = e^{g_r - g_i} in K and P: dq, dk and dg for rows r (+) and columns i (-),
//   dlog_alpha = reverse cumulative sum of dg over the chunk's rows,
//   dS = (s q gamma)^T dO + Diag(gamma_last) dS' - (k gamma)^T dr   (the previous chunk's dS').
//
// Every decay factor is a product of alphas (no e^{+g}): running products along the rows, or, in
// a chunk whose decay stays within e^-80, gamma_r times kappa_i / gamma_last (both bounded).
//
// Kernels: (1) one CTA per (sequence, head, d_v half of up to 64 columns) walks the chunks
// forward storing each chunk-start state (the checkpoints) with the chunk's r, u, K and T, then
// backward computing dv, dS0 and this half's share of dq, dk, dlog_alpha, dbeta, each chunk's
// inputs, checkpoint and stored terms prefetched (cp.async) while the chunk after it is
// computed; (2) a reduction adds the halves' shares in a fixed order (every d_v-side sum enters
// those gradients linearly) and writes them in their output types.  C = 16 keeps every chunk
// operand in shared memory at head size 128.
#include "kda_common.cuh"

namespace {

constexpr int kThreads = 512;
constexpr int kC = 16;
// A chunk whose decay stays within e^-80 in every channel (gamma_last >= e^-80) forms its decay
// factors D[r][i][c] = gamma_r / gamma_i as products of gamma_r and 1 / gamma_i, both in
// [1, e^80] or [e^-80, 1]: K, P and their gradients through D become plain small products.
constexpr float kFastGammaMin = 1.8048513e-35f;   // e^-80
// Floats of a checkpoint block: state [dk][dvh], r and u [kC][dvh], K and T [kC][kC + 1] (padded as
// in shared memory).
__host__ __device__ constexpr size_t kBlockFloats(int dk, int dvh) {
    return (size_t)(dk + 2 * kC) * dvh + 2 * kC * (kC + 1);
}
static_assert(kThreads == 32 * kC, "the K / P and gradient passes map warp w to row or column w, lane to a channel group");
static_assert(2 * 128 + 128 < kThreads - kC, "gradient products, rowsum, X and dbeta on separate threads");
static_assert(kC * kC <= kThreads && kC == 16, "dA: one thread per entry, a row per half-warp");

// Row pitches are padded to a multiple of 4 floats so that rows can be read 16 bytes at a time.
// ES is the input element size; the staging area at the end holds the next chunk's raw inputs
// (k, q, the gate, v, dO, beta), copied in while the current chunk is computed.
template <int DK, int DVH, int ES>
struct BwdLayout {
    static constexpr int LK = DK + 4, LV = DVH + 4, LC = kC + 1;
    // [kC][LK] arrays
    static constexpr int Q = 0, Kk = Q + kC * LK, AL = Kk + kC * LK, GA = AL + kC * LK, KA = GA + kC * LK,
                         KG = KA + kC * LK, SQ = KG + kC * LK, KK = SQ + kC * LK, DQ = KK + kC * LK,
                         DKc = DQ + kC * LK, DG = DKc + kC * LK;
    // [DK][LV] state and its gradient
    static constexpr int S = DG + kC * LK, DS = S + DK * LV;
    // [kC][LV] arrays
    static constexpr int V = DS + DK * LV, R = V + kC * LV, U = R + kC * LV, DO = U + kC * LV,
                         DU = DO + kC * LV, DR = DU + kC * LV;
    // [kC][LC] arrays
    static constexpr int KM = DR + kC * LV, TM = KM + kC * LC, PM = TM + kC * LC, DPM = PM + kC * LC,   // K, T adjacent
                         DTM = DPM + kC * LC, XM = DTM + kC * LC;
    static constexpr int GC = XM + kC * LC, BT = GC + DK, DB = BT + kC, DGC = DB + kC;
    static constexpr int DGP = DGC + DK;      // [kThreads / DK][DK] partial last-row g terms; while
                                              // a chunk's terms are formed, 1 / gamma_last at DGP + DK
    // staging, in bytes from its start: k, q [kC][DK] and v, dO [kC][DVH] in the input type, the
    // gate [kC][DK] fp32 (a scalar gate uses [kC]), beta [kC]
    static constexpr int ST = DGP + kThreads;
    static constexpr int ST_K = 0, ST_Q = ST_K + kC * DK * ES, ST_G = ST_Q + kC * DK * ES,
                         ST_V = ST_G + kC * DK * 4, ST_DO = ST_V + kC * DVH * ES, ST_B = ST_DO + kC * DVH * ES,
                         ST_BYTES = ST_B + kC * 4;
    static constexpr int floats = ST + ST_BYTES / 4;
    static constexpr size_t bytes = (size_t)floats * sizeof(float);
};

struct BwdArgs {
    KdaChunkArgs a;                 // forward inputs (gate form, flags 0)
    const void *dO;                 // [T_total, H, dv] dtype
    const float *dS_final;          // [N, H, dk, dv] or NULL
    void *dv_out;                   // [T_total, H, dv] dtype
    float *dS0;                     // [N, H, dk, dv] or NULL
    float *ckpt;                    // checkpoints: [max_chunks][H][nsplit] blocks of kBlockFloats(dk, dvh):
                                    // the chunk-start state, the chunk's r and u, then K and T
    float *part;                    // shares: [nsplit][T_total][H] x (3 dk + 1): dq, dk, dla, dbeta
    int64_t max_chunks;             // ceil(T_total / 16) + N with cu_seqlens, N ceil(T / 16) without
    int nsplit;
};

// Partial-gradient record of one token-head in a split's share: dq [dk], dk [dk], dla [dk], dbeta.
__device__ __forceinline__ size_t part_index(const BwdArgs &b, int split, size_t th, int dk) {
    return ((size_t)split * b.a.T_total * b.a.H + th) * (3 * (size_t)dk + 1);
}

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }

// Asynchronous global -> shared copies (16 bytes, or 4 for the strided per-token scalars).
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// acc += a . b over four consecutive k, in k order.
__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
    return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, fmaf(a.x, b.x, acc))));
}

template <typename Tin, int DK, int DVH>
__global__ void __launch_bounds__(kThreads, 1) kda_chunk_bwd_kernel(BwdArgs b) {   // 16 warps, <= 128 registers
    using L = BwdLayout<DK, DVH, (int)sizeof(Tin)>;
    constexpr int LK = L::LK, LV = L::LV, LC = L::LC, CH = kC;
    constexpr int RPT = kC * DVH / kThreads;   // rows per thread of the [C][dv] products
    constexpr int CPT = DK * DVH / kThreads;   // rows per thread of the [dk][dv] products
    constexpr int R7 = kC * DK / kThreads;     // rows per thread of the [C][dk] products
    static_assert(RPT >= 1 && (CPT % 4 == 0 || CPT < 4) && R7 >= 1 && DK % 32 == 0 && DVH % 4 == 0,
                  "backward tiling");
    constexpr int NTU = (DVH / 2) * (DK / 16);   // threads of the state updates (2 columns x 16 rows)
    static_assert(NTU + DK + kC <= kThreads, "state update tiling; the gradient write-out beside it");
    extern __shared__ float sm[];
    float *Q = sm + L::Q, *Kk = sm + L::Kk, *AL = sm + L::AL, *GA = sm + L::GA, *KA = sm + L::KA;
    float *KG = sm + L::KG, *SQ = sm + L::SQ, *KK = sm + L::KK, *DQ = sm + L::DQ, *DKc = sm + L::DKc;
    float *DG = sm + L::DG, *S = sm + L::S, *DS = sm + L::DS, *V = sm + L::V, *R = sm + L::R;
    float *U = sm + L::U, *DO = sm + L::DO, *DU = sm + L::DU, *DR = sm + L::DR;
    float *KM = sm + L::KM, *TM = sm + L::TM, *PM = sm + L::PM, *DPM = sm + L::DPM, *DTM = sm + L::DTM;
    float *XM = sm + L::XM, *GC = sm + L::GC, *BT = sm + L::BT, *DB = sm + L::DB, *DGC = sm + L::DGC;
    float *DGP = sm + L::DGP;
    float *RGC = DGP + DK;         // 1 / gamma_last of the chunk while its terms are formed (fast chunks)
    uint8_t *STG = reinterpret_cast<uint8_t *>(sm + L::ST);

    const KdaChunkArgs &a = b.a;
    const int H = a.H, dv = a.dv;
    const int split = blockIdx.x % b.nsplit, pair = blockIdx.x / b.nsplit;
    const int n = pair / H, h = pair % H;
    const int j0 = split * DVH;                 // first d_v column of this half
    const int tid = threadIdx.x;
    const float scale = a.scale;
    const Tin *qg = static_cast<const Tin *>(a.q);
    const Tin *kg = static_cast<const Tin *>(a.k);
    const Tin *vg = static_cast<const Tin *>(a.v);
    const Tin *dog = static_cast<const Tin *>(b.dO);
    Tin *dvg = static_cast<Tin *>(b.dv_out);

    int64_t t0, t1;
    kda::seq_bounds(a.cu_seqlens, n, a.T, a.T_total, t0, t1);
    // This sequence's first checkpoint chunk: the chunks of the sequences before it, the running
    // sum capped at max_chunks (offsets that are not non-decreasing can ask for more), and its
    // own chunk count capped to what is left: no checkpoint outside the workspace.
    int64_t base = 0;
    if (a.cu_seqlens) {
        for (int m = 0; m < n; ++m) {
            int64_t s0, s1;
            kda::seq_bounds(a.cu_seqlens, m, a.T, a.T_total, s0, s1);
            const int64_t want = (s1 - s0 + CH - 1) / CH;
            base += want < b.max_chunks - base ? want : b.max_chunks - base;
        }
    } else {
        base = (int64_t)n * ((a.T + CH - 1) / CH);
    }
    int64_t nch64 = (t1 - t0 + CH - 1) / CH;
    if (nch64 > b.max_chunks - base) nch64 = b.max_chunks - base;
    const int nch = (int)nch64;
    auto ckpt_block = [&](int ci) {
        return b.ckpt + (((size_t)(base + ci) * H + h) * b.nsplit + split) * kBlockFloats(DK, DVH);
    };
    // Copies rows of `rows` x DVH floats (packed, from global) into a padded shared array.
    auto copy_in = [&](float *dst, const float *src, int rows) {
        for (int q = tid; q < rows * DVH / 4; q += kThreads)
            cp_async16(dst + (4 * q / DVH) * LV + 4 * q % DVH, src + 4 * q);
    };
    const size_t sbase = (size_t)pair * DK * dv;

#pragma unroll 4
    for (int v4 = tid; v4 < DK * DVH / 4; v4 += kThreads) {
        const int c = 4 * v4 / DVH, j = 4 * v4 % DVH;
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4 *>(S + c * LV + j) = a.S0 ? ld4(a.S0 + sbase + (size_t)c * dv + j0 + j) : z;
        *reinterpret_cast<float4 *>(DS + c * LV + j) = b.dS_final ? ld4(b.dS_final + sbase + (size_t)c * dv + j0 + j) : z;
    }

    // Issues the copies of chunk c0's raw inputs into the staging area (rows < nr; q and dO
    // only for the backward pass).  Consumed by chunk_terms after a wait.
    auto prefetch = [&](int64_t c0, int nr, bool with_q) {
        constexpr int KCH = DK * (int)sizeof(Tin) / 16, GCH = DK * 4 / 16, VCH = DVH * (int)sizeof(Tin) / 16;
        for (int idx = tid; idx < nr * KCH; idx += kThreads) {
            const int r = idx / KCH, q16 = idx % KCH;
            const size_t off = ((size_t)(c0 + r) * H + h) * DK * sizeof(Tin) + 16 * q16;
            cp_async16(STG + L::ST_K + r * DK * (int)sizeof(Tin) + 16 * q16, reinterpret_cast<const uint8_t *>(kg) + off);
            if (with_q)
                cp_async16(STG + L::ST_Q + r * DK * (int)sizeof(Tin) + 16 * q16,
                           reinterpret_cast<const uint8_t *>(qg) + off);
        }
        if (a.gate_kind == kda::GATE_CHANNEL) {
            for (int idx = tid; idx < nr * GCH; idx += kThreads) {
                const int r = idx / GCH, q16 = idx % GCH;
                cp_async16(STG + L::ST_G + r * DK * 4 + 16 * q16,
                           static_cast<const uint8_t *>(a.gate) + ((size_t)(c0 + r) * H + h) * DK * 4 + 16 * q16);
            }
        } else if (a.gate_kind == kda::GATE_SCALAR && tid < nr) {
            cp_async4(STG + L::ST_G + 4 * tid, static_cast<const float *>(a.gate) + (size_t)(c0 + tid) * H + h);
        }
        for (int idx = tid; idx < nr * VCH; idx += kThreads) {
            const int r = idx / VCH, q16 = idx % VCH;
            const size_t off = (((size_t)(c0 + r) * H + h) * dv + j0) * sizeof(Tin) + 16 * q16;
            cp_async16(STG + L::ST_V + r * DVH * (int)sizeof(Tin) + 16 * q16, reinterpret_cast<const uint8_t *>(vg) + off);
            if (with_q)
                cp_async16(STG + L::ST_DO + r * DVH * (int)sizeof(Tin) + 16 * q16,
                           reinterpret_cast<const uint8_t *>(dog) + off);
        }
        if (tid < nr) cp_async4(STG + L::ST_B + 4 * tid, a.beta + (size_t)(c0 + tid) * H + h);
        cp_async_commit();
    };
    __syncthreads();

    // Takes chunk c0's rows from the staging area (zeros / alpha = 1 / beta = 0 past the sequence
    // end; with_q: also q and dO), starts the copies of the next chunk (pf_nr rows from pf_c0,
    // none when pf_nr = 0), and forms the decay products and the chunk matrices K, T, P.
    // The forward pass (form_ru) forms K, T, r and u; the backward pass (with_q) forms P and finds
    // K, T, r and u in place (stored by the forward pass with the checkpoint, prefetched).
    auto chunk_terms = [&](int64_t c0, int nr, bool with_q, int64_t pf_c0, int pf_nr, bool pf_q,
                           bool form_ru) -> bool {
        cp_async_wait_all();
        __syncthreads();                       // this chunk's staged rows are visible to all
        {
            const Tin *sk = reinterpret_cast<const Tin *>(STG + L::ST_K), *sq = reinterpret_cast<const Tin *>(STG + L::ST_Q);
            const Tin *sv = reinterpret_cast<const Tin *>(STG + L::ST_V), *sdo = reinterpret_cast<const Tin *>(STG + L::ST_DO);
            const float *sg = reinterpret_cast<const float *>(STG + L::ST_G), *sb = reinterpret_cast<const float *>(STG + L::ST_B);
#pragma unroll
            for (int it = 0; it < CH * DK / kThreads; ++it) {
                const int idx = tid + it * kThreads, r = idx / DK, c = idx % DK;
                float kv = 0.f, qv = 0.f, al = 1.f;
                if (r < nr) {
                    kv = kda::to_f32(sk[r * DK + c]);
                    qv = with_q ? kda::to_f32(sq[r * DK + c]) : 0.f;
                    const float la = a.gate_kind == kda::GATE_CHANNEL ? sg[r * DK + c]
                                     : (a.gate_kind == kda::GATE_SCALAR ? sg[r] : 0.f);
                    al = expf(la);
                }
                Kk[r * LK + c] = kv;
                Q[r * LK + c] = qv;
                AL[r * LK + c] = al;
            }
#pragma unroll
            for (int it = 0; it < CH * DVH / kThreads; ++it) {
                const int idx = tid + it * kThreads, r = idx / DVH, j = idx % DVH;
                V[r * LV + j] = r < nr ? kda::to_f32(sv[r * DVH + j]) : 0.f;
                if (with_q) DO[r * LV + j] = r < nr ? kda::to_f32(sdo[r * DVH + j]) : 0.f;
            }
            if (tid < CH) BT[tid] = tid < nr ? sb[tid] : 0.f;
        }
        __syncthreads();                       // the staging area is free
        if (pf_nr > 0) prefetch(pf_c0, pf_nr, pf_q);
        // gamma (forward running product) and kappa (reverse), per channel
        for (int c = tid; c < DK; c += kThreads) {
            float g = 1.f;
#pragma unroll
            for (int r = 0; r < CH; ++r) {
                g *= AL[r * LK + c];
                GA[r * LK + c] = g;
                KG[r * LK + c] = Kk[r * LK + c] * g;
                SQ[r * LK + c] = scale * Q[r * LK + c] * g;
            }
            GC[c] = g;
            RGC[c] = 1.f / g;
            float kp = 1.f;
#pragma unroll
            for (int r = CH - 1; r >= 0; --r) {
                KA[r * LK + c] = kp;
                KK[r * LK + c] = Kk[r * LK + c] * kp;
                kp *= AL[r * LK + c];
            }
        }
        const bool fast = __syncthreads_and(tid >= DK || GC[tid] >= kFastGammaMin);
        if (fast) {
            // K = (k gamma)(k kappa / gamma_last)^T, P = (s q gamma)(k kappa / gamma_last)^T (lower
            // parts).  Thread: (row r, column i).
            if (tid < CH * CH) {
                const int r = tid / CH, i = tid % CH;
                const float *A = form_ru ? KG : SQ;    // K in the forward pass, P in the backward
                float acc = 0.f;
                if (i <= r) {
#pragma unroll 4
                    for (int c = 0; c < DK; c += 4) {
                        const float4 kk = ld4(KK + i * LK + c), rg = ld4(RGC + c);
                        const float4 ki = make_float4(kk.x * rg.x, kk.y * rg.y, kk.z * rg.z, kk.w * rg.w);
                        acc = dot4(ld4(A + r * LK + c), ki, acc);
                    }
                }
                if (form_ru) KM[r * LC + i] = r > i ? acc : 0.f;
                else PM[r * LC + i] = r >= i ? acc : 0.f;
            }
        } else {
        // K and P: warp i, lane = channel group cg of 32, carries running products down the rows
        // r >= i; the 32 groups of a column are then summed by full-warp shuffles, all rows'
        // sums together (every lane of the warp takes part).
            const int i = tid >> 5, cg = tid & 31;
            constexpr int CPT = DK / 32;
            float f[CPT], sk[CH], sp[CH];
#pragma unroll
            for (int m = 0; m < CPT; ++m) f[m] = 1.f;
#pragma unroll
            for (int r = 0; r < CH; ++r) {
                sk[r] = 0.f;
                sp[r] = 0.f;
                if (r >= i) {
#pragma unroll
                    for (int m = 0; m < CPT; ++m) {
                        const int c = cg + 32 * m;
                        if (r > i) f[m] *= AL[r * LK + c];
                        const float kd = Kk[i * LK + c] * f[m];
                        sk[r] = fmaf(Kk[r * LK + c], kd, sk[r]);
                        sp[r] = fmaf(Q[r * LK + c], kd, sp[r]);
                    }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
                for (int r = 0; r < CH; ++r) {
                    sk[r] += __shfl_xor_sync(0xffffffffu, sk[r], o);
                    sp[r] += __shfl_xor_sync(0xffffffffu, sp[r], o);
                }
            }
            if (cg == 0) {
#pragma unroll
                for (int r = 0; r < CH; ++r) {
                    if (form_ru) KM[r * LC + i] = r > i ? sk[r] : 0.f;
                    if (with_q) PM[r * LC + i] = r >= i ? scale * sp[r] : 0.f;
                }
            }
        }
        __syncthreads();
        // T = (I + Diag(beta) K)^{-1}, unit lower triangular: column i by forward substitution,
        // the column in registers (its entries above row i are zero, so the sums over m < i add
        // exact zeros before the first term, as if they started at m = i)
        if (form_ru && tid < CH) {
            const int i = tid;
            float t[CH];
#pragma unroll
            for (int r = 0; r < CH; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < r; ++m) acc = fmaf(BT[r] * KM[r * LC + m], t[m], acc);
                t[r] = r < i ? 0.f : (r == i ? 1.f : -acc);
                TM[r * LC + i] = t[r];
            }
        }
        __syncthreads();
        // r = v - (k gamma) S (thread: column j, 4 rows, so each state value feeds 4 rows); then
        // u = T Diag(beta) r (thread: column j, RPT rows).  The backward pass finds both in place
        // (the forward pass stored them with the checkpoint).
        if (form_ru) {
            if (tid < 4 * DVH) {
                const int j = tid % DVH, r0 = (tid / DVH) * 4;
                float acc[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) acc[t] = V[(r0 + t) * LV + j];
                for (int c = 0; c < DK; c += 4) {
                    const float4 s4 = make_float4(S[c * LV + j], S[(c + 1) * LV + j], S[(c + 2) * LV + j],
                                                  S[(c + 3) * LV + j]);
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const float4 kg = ld4(KG + (r0 + t) * LK + c);
                        acc[t] = dot4(make_float4(-kg.x, -kg.y, -kg.z, -kg.w), s4, acc[t]);
                    }
                }
#pragma unroll
                for (int t = 0; t < 4; ++t) R[(r0 + t) * LV + j] = acc[t];
            }
            __syncthreads();
            const int j = tid % DVH, r0 = (tid / DVH) * RPT;
#pragma unroll
            for (int t = 0; t < RPT; ++t) {
                const int r = r0 + t;
                float u = 0.f;
                for (int i = 0; i <= r; ++i) u = fmaf(TM[r * LC + i] * BT[i], R[i * LV + j], u);
                U[r * LV + j] = u;
            }
        }
        __syncthreads();
        return fast;
    };

    // ---------------------------------------------------------------- forward: checkpoints
    auto chunk_rows = [&](int ci) { const int64_t c0 = t0 + (int64_t)ci * CH; return (int)(t1 - c0 < CH ? t1 - c0 : CH); };
    if (nch > 0) prefetch(t0, chunk_rows(0), false);
    for (int ci = 0; ci < nch; ++ci) {
        const int64_t c0 = t0 + (int64_t)ci * CH;
        const int nr = chunk_rows(ci);
        float *dst = ckpt_block(ci);
#pragma unroll 4
        for (int v4 = tid; v4 < DK * DVH / 4; v4 += kThreads)
            *reinterpret_cast<float4 *>(dst + 4 * v4) = ld4(S + (4 * v4 / DVH) * LV + 4 * v4 % DVH);
        // next: chunk ci + 1, or after the last one the backward pass's first chunk (the last)
        const int nx = ci + 1 < nch ? ci + 1 : nch - 1;
        chunk_terms(c0, nr, false, t0 + (int64_t)nx * CH, chunk_rows(nx), ci + 1 >= nch, true);
        {   // the chunk's r, u, K and T beside its checkpoint, for the backward pass
            float *ru = dst + DK * DVH;
            for (int q = tid; q < 2 * CH * DVH / 4; q += kThreads) {
                const int row = 4 * q / DVH, j = 4 * q % DVH;
                const float *from = row < CH ? R + row * LV + j : U + (row - CH) * LV + j;
                *reinterpret_cast<float4 *>(ru + 4 * q) = ld4(from);
            }
            float *kt = ru + 2 * CH * DVH;         // K and T, contiguous in shared memory
            for (int q = tid; q < 2 * CH * LC / 4; q += kThreads) *reinterpret_cast<float4 *>(kt + 4 * q) = ld4(KM + 4 * q);
        }
        // S <- Diag(gamma_last) S + (k kappa)^T u, in place.  Thread: columns j, j + 1 and 16 rows
        // (each broadcast (k kappa) value feeds both columns).
        if (tid < NTU) {
            const int j = 2 * (tid % (DVH / 2)), c0 = (tid / (DVH / 2)) * 16;
            float2 acc[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const float g = GC[c0 + t];
                const float2 x = *reinterpret_cast<const float2 *>(S + (c0 + t) * LV + j);
                acc[t] = make_float2(g * x.x, g * x.y);
            }
            for (int r = 0; r < CH; ++r) {
                const float2 u = *reinterpret_cast<const float2 *>(U + r * LV + j);
#pragma unroll
                for (int t = 0; t < 16; t += 4) {
                    const float4 kk = ld4(KK + r * LK + c0 + t);
                    const float kv[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc[t + e].x = fmaf(kv[e], u.x, acc[t + e].x);
                        acc[t + e].y = fmaf(kv[e], u.y, acc[t + e].y);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < 16; ++t) *reinterpret_cast<float2 *>(S + (c0 + t) * LV + j) = acc[t];
        }
        __syncthreads();
    }

    // ---------------------------------------------------------------- backward
    // Each chunk's checkpoint, r, u, K and T arrive by cp.async: the last chunk's checkpoint now
    // (its r, u, K and T are still in place from the forward pass), every earlier chunk's once the
    // chunk after it no longer reads them (below: S, R, U after the gradient products, K and T after
    // dA).
    if (nch > 0) {
        copy_in(S, ckpt_block(nch - 1), DK);
        cp_async_commit();
    }
    for (int ci = nch - 1; ci >= 0; --ci) {
        const int64_t c0 = t0 + (int64_t)ci * CH;
        const int nr = (int)(t1 - c0 < CH ? t1 - c0 : CH);
        const bool fast = chunk_terms(c0, nr, true, c0 - CH, ci > 0 ? CH : 0, true, false);

        // du = P^T dO + (k kappa) dS', then dr = Diag(beta) T^T du (this half's dv rows).
        {
            if (tid < 4 * DVH) {                   // du: thread column j, 4 rows
                const int j = tid % DVH, i0 = (tid / DVH) * 4;
                float acc[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int i = i0 + t;
                    float a0 = 0.f;
                    for (int r = i; r < CH; ++r) a0 = fmaf(PM[r * LC + i], DO[r * LV + j], a0);
                    acc[t] = a0;
                }
                for (int c = 0; c < DK; c += 4) {
                    const float4 d4 = make_float4(DS[c * LV + j], DS[(c + 1) * LV + j], DS[(c + 2) * LV + j],
                                                  DS[(c + 3) * LV + j]);
#pragma unroll
                    for (int t = 0; t < 4; ++t) acc[t] = dot4(ld4(KK + (i0 + t) * LK + c), d4, acc[t]);
                }
#pragma unroll
                for (int t = 0; t < 4; ++t) DU[(i0 + t) * LV + j] = acc[t];
            }
            __syncthreads();
            const int j = tid % DVH, i0 = (tid / DVH) * RPT;   // dr: thread column j, RPT rows
#pragma unroll
            for (int t = 0; t < RPT; ++t) {
                const int i = i0 + t;
                float a1 = 0.f;
                for (int r = i; r < CH; ++r) a1 = fmaf(TM[r * LC + i], DU[r * LV + j], a1);
                a1 *= BT[i];
                DR[i * LV + j] = a1;
                if (i < nr) dvg[((size_t)(c0 + i) * H + h) * dv + j0 + j] = kda::from_f32<Tin>(a1);
            }
        }
        // dP = tril(dO u^T) and dT' = tril(du r^T) over this half's columns
        for (int idx = tid; idx < CH * CH; idx += kThreads) {
            const int r = idx / CH, i = idx % CH;
            float p = 0.f, t = 0.f;
            if (i <= r) {
                for (int j = 0; j < DVH; j += 4) {
                    p = dot4(ld4(DO + r * LV + j), ld4(U + i * LV + j), p);
                    t = dot4(ld4(DU + r * LV + j), ld4(R + i * LV + j), t);
                }
            }
            DPM[r * LC + i] = p;
            DTM[r * LC + i] = t;
        }
        __syncthreads();
        // the decay-weighted elementwise terms: d(s q gamma) = dO S^T, d(k gamma) = -dr S^T,
        // d(k kappa) = u dS'^T, and the last row's g terms.  Thread: channels c and c + DK / 2, 4 rows
        // (each broadcast row of dO, dr, u feeds both channels); beside them other warps form
        // gamma_last rowsum(dS' * S) and dbeta from T' = T Diag(beta).
        {
            constexpr int NTH = 2 * DK;
            if (tid < NTH) {
                const int cp = tid % (DK / 2), g4 = tid / (DK / 2), r0 = 4 * g4;
                const int cc[2] = {cp, cp + DK / 2};
                float dsq[2][4], dkg[2][4], dkk[2][4];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int t = 0; t < 4; ++t) dsq[hh][t] = dkg[hh][t] = dkk[hh][t] = 0.f;
                for (int j = 0; j < DVH; j += 4) {
                    const float4 s0 = ld4(S + cc[0] * LV + j), s1 = ld4(S + cc[1] * LV + j);
                    const float4 d0 = ld4(DS + cc[0] * LV + j), d1 = ld4(DS + cc[1] * LV + j);
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int r = r0 + t;
                        const float4 o4 = ld4(DO + r * LV + j), dr = ld4(DR + r * LV + j), u4 = ld4(U + r * LV + j);
                        const float4 nd = make_float4(-dr.x, -dr.y, -dr.z, -dr.w);
                        dsq[0][t] = dot4(o4, s0, dsq[0][t]);
                        dsq[1][t] = dot4(o4, s1, dsq[1][t]);
                        dkg[0][t] = dot4(nd, s0, dkg[0][t]);
                        dkg[1][t] = dot4(nd, s1, dkg[1][t]);
                        dkk[0][t] = dot4(u4, d0, dkk[0][t]);
                        dkk[1][t] = dot4(u4, d1, dkk[1][t]);
                    }
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int c = cc[hh];
                    float kkp = 0.f;
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int o = (r0 + t) * LK + c;
                        DQ[o] = scale * GA[o] * dsq[hh][t];
                        DKc[o] = GA[o] * dkg[hh][t] + KA[o] * dkk[hh][t];
                        DG[o] = dsq[hh][t] * SQ[o] + dkg[hh][t] * KG[o] - dkk[hh][t] * KK[o];
                        kkp = fmaf(dkk[hh][t], KK[o], kkp);
                    }
                    DGP[g4 * DK + c] = kkp;           // summed over the 4 row groups below, in order
                }
            } else if (tid < NTH + DK) {
                const int c = tid - NTH;
                float gl = 0.f;
                for (int j = 0; j < DVH; j += 4) gl = dot4(ld4(DS + c * LV + j), ld4(S + c * LV + j), gl);
                DGC[c] = GC[c] * gl;
            }
            if (tid >= kThreads - CH) {
                const int i = tid - (kThreads - CH);
                float acc = 0.f;
                for (int r = i; r < CH; ++r) acc = fmaf(DTM[r * LC + i], TM[r * LC + i], acc);
                DB[i] = acc;
            } else if (tid >= NTH + DK) {        // X = dT' Diag(beta) T^T
                for (int idx = tid - (NTH + DK); idx < CH * CH; idx += kThreads - CH - NTH - DK) {
                    const int r = idx / CH, m = idx % CH;
                    float acc = 0.f;
                    for (int i = 0; i <= (r < m ? r : m); ++i)
                        acc = fmaf(DTM[r * LC + i] * BT[i], TM[m * LC + i], acc);
                    XM[r * LC + m] = acc;
                }
            }
        }
        __syncthreads();
        if (ci > 0) {                          // S, R and U are not read again for this chunk
            const float *src = ckpt_block(ci - 1);
            copy_in(S, src, DK);
            copy_in(R, src + DK * DVH, CH);
            copy_in(U, src + (DK + CH) * DVH, CH);
            cp_async_commit();
        }
        // The last row's g terms summed; dA = strict-lower(-T^T X) (X = dT T^T, dT = dT' Diag(beta),
        // formed beside the gradient products), dbeta_p += sum_m dA_pm K_pm (the 16 threads of row p
        // are a half-warp: shuffles), dK = Diag(beta) dA into DTM.
        for (int c = tid; c < DK; c += kThreads) {
            float acc = DGC[c];
            for (int g = 0; g < CH / 4; ++g) acc += DGP[g * DK + c];
            DGC[c] = acc;                     // both go to the last row's g
        }
        if (tid < CH * CH) {
            const int p = tid / CH, m = tid % CH;
            float acc = 0.f;
            if (m < p)
                for (int r = p; r < CH; ++r) acc = fmaf(TM[r * LC + p], XM[r * LC + m], acc);
            const float da = -acc;               // dA, strictly lower (zero elsewhere)
            float t = m < p ? da * KM[p * LC + m] : 0.f;
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
            if (m == 0) DB[p] += t;
            DTM[p * LC + m] = da * BT[p];        // dK
        }
        __syncthreads();
        if (ci > 0) {                          // K and T are not read again for this chunk
            const float *kt = ckpt_block(ci - 1) + (DK + 2 * CH) * DVH;
            for (int q = tid; q < 2 * CH * LC / 4; q += kThreads) cp_async16(KM + 4 * q, kt + 4 * q);
            cp_async_commit();
        }
        if (fast) {
            // through D = gamma_r / gamma_i in K and P, as products: for row / column x and channel c
            //   adk = (1 / gamma_x) sum_r (dP_rx (s q gamma)_r + dK_rx (k gamma)_r),  adg = -k_x adk,
            //   bdq = s (gamma_x / gamma_last) sum_i dP_xi (k kappa)_i,  bdk likewise with dK,
            //   bdg = q_x bdq + k_x bdk.
            // Thread: rows x and x + 8, channels c .. c + 3.
            constexpr int C4 = DK / 4;
            if (tid < 8 * C4) {
                const int xa = tid / C4, c = 4 * (tid % C4);
                float4 a[2] = {}, b1[2] = {}, b2[2] = {};
#pragma unroll
                for (int r = 0; r < CH; ++r) {
                    const float4 sq = ld4(SQ + r * LK + c), kg = ld4(KG + r * LK + c), kk = ld4(KK + r * LK + c);
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const int x = xa + 8 * h2;
                        const float pc = DPM[r * LC + x], kc = DTM[r * LC + x], pr = DPM[x * LC + r], kr = DTM[x * LC + r];
                        a[h2].x = fmaf(pc, sq.x, fmaf(kc, kg.x, a[h2].x));
                        a[h2].y = fmaf(pc, sq.y, fmaf(kc, kg.y, a[h2].y));
                        a[h2].z = fmaf(pc, sq.z, fmaf(kc, kg.z, a[h2].z));
                        a[h2].w = fmaf(pc, sq.w, fmaf(kc, kg.w, a[h2].w));
                        b1[h2].x = fmaf(pr, kk.x, b1[h2].x);
                        b1[h2].y = fmaf(pr, kk.y, b1[h2].y);
                        b1[h2].z = fmaf(pr, kk.z, b1[h2].z);
                        b1[h2].w = fmaf(pr, kk.w, b1[h2].w);
                        b2[h2].x = fmaf(kr, kk.x, b2[h2].x);
                        b2[h2].y = fmaf(kr, kk.y, b2[h2].y);
                        b2[h2].z = fmaf(kr, kk.z, b2[h2].z);
                        b2[h2].w = fmaf(kr, kk.w, b2[h2].w);
                    }
                }
                const float4 gc = ld4(GC + c);     // RGC's space is taken by the g terms by now
                const float rgv[4] = {1.f / gc.x, 1.f / gc.y, 1.f / gc.z, 1.f / gc.w};
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int x = xa + 8 * h2, o = x * LK + c;
                    const float4 ka = ld4(KA + o), ga = ld4(GA + o), kx = ld4(Kk + o), qx = ld4(Q + o);
                    const float kav[4] = {ka.x, ka.y, ka.z, ka.w}, gav[4] = {ga.x, ga.y, ga.z, ga.w};
                    const float kxv[4] = {kx.x, kx.y, kx.z, kx.w}, qxv[4] = {qx.x, qx.y, qx.z, qx.w};
                    const float av[4] = {a[h2].x, a[h2].y, a[h2].z, a[h2].w};
                    const float b1v[4] = {b1[h2].x, b1[h2].y, b1[h2].z, b1[h2].w};
                    const float b2v[4] = {b2[h2].x, b2[h2].y, b2[h2].z, b2[h2].w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float adk = kav[j] * rgv[j] * av[j];
                        const float gr = gav[j] * rgv[j];
                        const float bdq = scale * gr * b1v[j], bdk = gr * b2v[j];
                        DQ[o + j] += bdq;
                        DKc[o + j] += adk + bdk;
                        DG[o + j] += -kxv[j] * adk + (qxv[j] * bdq + kxv[j] * bdk);
                    }
                }
            }
        } else {
        // through D = e^{g_r - g_i} in K and P: warp x, lane = channel group cg; as column i = x
        // it walks rows r >= x, as row r = x it walks columns i <= x, each with running products.
            const int x = tid >> 5, cg = tid & 31;
            constexpr int CPT = DK / 32;
#pragma unroll
            for (int m = 0; m < CPT; ++m) {
                const int c = cg + 32 * m;
                const float kx = Kk[x * LK + c], qx = Q[x * LK + c];
                float f = 1.f, adk = 0.f, adg = 0.f;
                for (int r = x; r < CH; ++r) {                    // x as the column i
                    if (r > x) f *= AL[r * LK + c];
                    const float w = scale * DPM[r * LC + x] * Q[r * LK + c] +
                                    (r > x ? DTM[r * LC + x] * Kk[r * LK + c] : 0.f);
                    adk = fmaf(f, w, adk);
                    adg = fmaf(-f * w, kx, adg);
                }
                float g = 1.f, bdq = 0.f, bdk = 0.f, bdg = 0.f;
                for (int i = x; i >= 0; --i) {                    // x as the row r
                    if (i < x) g *= AL[(i + 1) * LK + c];
                    const float ki = Kk[i * LK + c];
                    const float dp = DPM[x * LC + i], dkk = i < x ? DTM[x * LC + i] : 0.f;
                    bdq = fmaf(scale * dp * ki, g, bdq);
                    bdk = fmaf(dkk * ki, g, bdk);
                    bdg = fmaf(g * ki, scale * dp * qx + dkk * kx, bdg);
                }
                DQ[x * LK + c] += bdq;
                DKc[x * LK + c] += adk + bdk;
                DG[x * LK + c] += adg + bdg;
            }
        }
        __syncthreads();
        // dlog_alpha = reverse cumulative sum of dg; write this half's share of the rows (on the
        // threads past those of the dS update below, which runs at the same time)
        if (tid >= NTU && tid < NTU + DK) {
            const int c = tid - NTU;
            float acc = DGC[c];                    // the last row's extra g terms
            for (int r = CH - 1; r >= 0; --r) {
                acc += DG[r * LK + c];
                if (r < nr) {
                    const size_t th = (size_t)(c0 + r) * H + h;
                    float *rec = b.part + part_index(b, split, th, DK);
                    rec[c] = DQ[r * LK + c];
                    rec[DK + c] = DKc[r * LK + c];
                    rec[2 * DK + c] = acc;
                }
            }
        }
        if (tid >= NTU + DK && tid < NTU + DK + nr) {
            const int r = tid - NTU - DK;
            b.part[part_index(b, split, (size_t)(c0 + r) * H + h, DK) + 3 * DK] = DB[r];
        }
        // dS for the previous chunk, in place: (s q gamma)^T dO + Diag(gamma_last) dS' - (k gamma)^T dr.
        // Thread: columns j, j + 1 and 16 rows.
        if (tid < NTU) {
            const int j = 2 * (tid % (DVH / 2)), cb = (tid / (DVH / 2)) * 16;
            float2 acc[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const float g = GC[cb + t];
                const float2 x = *reinterpret_cast<const float2 *>(DS + (cb + t) * LV + j);
                acc[t] = make_float2(g * x.x, g * x.y);
            }
            for (int r = 0; r < CH; ++r) {
                const float2 d = *reinterpret_cast<const float2 *>(DO + r * LV + j);
                const float2 e2 = *reinterpret_cast<const float2 *>(DR + r * LV + j);
#pragma unroll
                for (int t = 0; t < 16; t += 4) {
                    const float4 sq = ld4(SQ + r * LK + cb + t), kg = ld4(KG + r * LK + cb + t);
                    const float sv[4] = {sq.x, sq.y, sq.z, sq.w}, gv[4] = {kg.x, kg.y, kg.z, kg.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc[t + e].x = fmaf(sv[e], d.x, fmaf(-gv[e], e2.x, acc[t + e].x));
                        acc[t + e].y = fmaf(sv[e], d.y, fmaf(-gv[e], e2.y, acc[t + e].y));
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < 16; ++t) *reinterpret_cast<float2 *>(DS + (cb + t) * LV + j) = acc[t];
        }
        __syncthreads();
    }
    if (b.dS0)
#pragma unroll 4
        for (int v4 = tid; v4 < DK * DVH / 4; v4 += kThreads) {
            const int c = 4 * v4 / DVH, j = 4 * v4 % DVH;
            *reinterpret_cast<float4 *>(b.dS0 + sbase + (size_t)c * dv + j0 + j) = ld4(DS + c * LV + j);
        }
}

// Adds the halves' shares in split order and writes dq, dk (input dtype), the gate gradient
// (per channel, or summed over channels for the scalar gate) and dbeta.  One warp per
// token-head.
template <typename Tin>
__global__ void kda_chunk_bwd_reduce_kernel(BwdArgs b, void *dq_out, void *dk_out, float *dgate, float *dbeta) {
    const int dk = b.a.dk;
    const size_t rows = (size_t)b.a.T_total * b.a.H;
    const size_t th = (size_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    if (th >= rows) return;
    Tin *dq = static_cast<Tin *>(dq_out), *dkp = static_cast<Tin *>(dk_out);
    float gsum = 0.f;
    for (int c = lane; c < dk; c += 32) {
        float sq = 0.f, sk = 0.f, sg = 0.f;
        for (int s = 0; s < b.nsplit; ++s) {
            const float *rec = b.part + part_index(b, s, th, dk);
            sq += rec[c];
            sk += rec[dk + c];
            sg += rec[2 * dk + c];
        }
        dq[th * dk + c] = kda::from_f32<Tin>(sq);
        dkp[th * dk + c] = kda::from_f32<Tin>(sk);
        if (b.a.gate_kind == kda::GATE_CHANNEL && dgate) dgate[th * dk + c] = sg;
        gsum += sg;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) gsum += __shfl_xor_sync(0xffffffffu, gsum, o);
    if (lane == 0) {
        float sb = 0.f;
        for (int s = 0; s < b.nsplit; ++s) sb += b.part[part_index(b, s, th, dk) + 3 * dk];
        dbeta[th] = sb;
        if (b.a.gate_kind == kda::GATE_SCALAR && dgate) dgate[th] = gsum;
    }
}

template <typename Tin, int DK, int DVH>
cudaError_t launch_bwd(const BwdArgs &b, cudaStream_t st) {
    const size_t smem = BwdLayout<DK, DVH, (int)sizeof(Tin)>::bytes;
    cudaError_t e = cudaFuncSetAttribute(kda_chunk_bwd_kernel<Tin, DK, DVH>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((int64_t)b.a.N * b.a.H * b.nsplit);
    kda_chunk_bwd_kernel<Tin, DK, DVH><<<grid, kThreads, smem, st>>>(b);
    return cudaGetLastError();
}

template <typename Tin, int DK>
cudaError_t pick_dvh(const BwdArgs &b, cudaStream_t st) {
    switch (b.a.dv) {
    case 32: return launch_bwd<Tin, DK, 32>(b, st);
    case 64:
    case 128: return launch_bwd<Tin, DK, 64>(b, st);
    }
    return cudaErrorInvalidValue;
}

template <typename Tin>
cudaError_t run(const BwdArgs &b, void *dq, void *dk, float *dgate, float *dbeta, cudaStream_t st) {
    cudaError_t e;
    switch (b.a.dk) {
    case 32: e = pick_dvh<Tin, 32>(b, st); break;
    case 64: e = pick_dvh<Tin, 64>(b, st); break;
    case 128: e = pick_dvh<Tin, 128>(b, st); break;
    default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    const size_t rows = (size_t)b.a.T_total * b.a.H;
    if (rows == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((rows + 7) / 8);
    kda_chunk_bwd_reduce_kernel<Tin><<<blocks, 256, 0, st>>>(b, dq, dk, dgate, dbeta);
    return cudaGetLastError();
}

}  // namespace

namespace {
int64_t bwd_max_chunks(const KdaChunkArgs &a) {
    return a.cu_seqlens ? (a.T_total + kC - 1) / kC + a.N : (int64_t)a.N * ((a.T + kC - 1) / kC);
}
}  // namespace

size_t kda_chunk_bwd_workspace_bytes(const KdaChunkArgs &a) {
    const int nsplit = a.dv > 64 ? a.dv / 64 : 1, dvh = a.dv / nsplit;
    const size_t ck = (size_t)bwd_max_chunks(a) * a.H * nsplit * kBlockFloats(a.dk, dvh) * sizeof(float);
    const size_t part = (size_t)nsplit * a.T_total * a.H * (3 * (size_t)a.dk + 1) * sizeof(float);
    return ((ck + 255) & ~(size_t)255) + part;
}

cudaError_t kda_launch_chunk_bwd(const KdaChunkArgs &a, int dtype, const void *dO, const float *dS_final,
                                 void *dq, void *dk, void *dv, float *dgate, float *dbeta, float *dS0,
                                 void *ws, cudaStream_t stream) {
    BwdArgs b;
    b.a = a;
    b.dO = dO;
    b.dS_final = dS_final;
    b.dv_out = dv;
    b.dS0 = dS0;
    b.nsplit = a.dv > 64 ? a.dv / 64 : 1;
    const int dvh = a.dv / b.nsplit;
    b.max_chunks = bwd_max_chunks(a);
    const size_t ck = (size_t)b.max_chunks * a.H * b.nsplit * kBlockFloats(a.dk, dvh) * sizeof(float);
    b.ckpt = static_cast<float *>(ws);
    b.part = reinterpret_cast<float *>(static_cast<char *>(ws) + ((ck + 255) & ~(size_t)255));
    return dtype == 0 ? run<float>(b, dq, dk, dgate, dbeta, stream) : run<__nv_bfloat16>(b, dq, dk, dgate, dbeta, stream);
}
