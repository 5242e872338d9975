// Chunked KDA prefill in fp32 SIMT arithmetic (the KDA_F32 path).
//
// The WY/UT chunk algorithm of "22,580" §6.3 with the per-channel cumulative
// decay of its §08/§9.1, for chunks of C = 64 tokens.  Per chunk, with the
// decay factor of a pair of rows i <= r written as the product of the
// per-channel decays strictly after i up to r, D[r][i][c] = prod_{i<s<=r}
// alpha[s][c], the query scale s, and the state S (dk x dv) carried across
// chunks:
//
//   A[r][i] = beta_r sum_c k[r][c] k[i][c] D[r][i][c]     i < r
//   P[r][i] = s      sum_c q[r][c] k[i][c] D[r][i][c]     i <= r
//   T'      = (I + A)^{-1} Diag(beta)                  forward substitution
//   W = T' (k gamma),  U = T' v,  u = U - W S          gamma[r] = prod_{s<=r} alpha[s]
//   o = (s q gamma) S + P u
//   S <- Diag(gamma_last) S + (k kappa)^T u            kappa[r] = prod_{s>r} alpha[s]
//
// Every decay factor is a product of alphas in (0, 1], computed by running
// products: no factor can overflow, and none loses digits to the cancellation
// of two large cumulative log-decays (log_alpha as strong as -1e4 mixed with
// ordinary values stays exact to fp32 rounding).  One CTA of 256 threads per
// (sequence, head).  The state lives in registers: thread (j, sl) holds column
// j of rows [sl*RW, (sl+1)*RW).  All chunk operands live in shared memory with
// padded (odd) row strides.  This path favours exactness and simplicity over
// speed.
#pragma once
#include "kda_common.cuh"

namespace kda_simt {

constexpr int kSimtThreads = 256;
constexpr int kChunk = 64;

template <int DK, int DV>
struct SimtLayout {
    static constexpr int NSL = kSimtThreads / DV;   // slices of the state rows
    static constexpr int RW = DK / NSL;             // state rows per thread
    static constexpr int RU = kChunk / NSL;         // chunk rows of u / o per thread
    static constexpr int LK = DK + 1, LV = DV + 1, LC = kChunk + 1;
    static constexpr int LKV = LK > LV ? LK : LV;
    static constexpr size_t floats =
        (size_t)kChunk * LKV + 3 * (size_t)kChunk * LK + (size_t)kChunk * LV +
        3 * (size_t)kChunk * LC + kChunk + DK;
    static constexpr size_t bytes = floats * sizeof(float);
    static_assert(kSimtThreads % DV == 0 && DK % NSL == 0 && kChunk % NSL == 0, "tiling");
};

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kSimtThreads, 1) kda_chunk_simt_kernel(KdaChunkArgs a) {
    using L = SimtLayout<DK, DV>;
    constexpr int CH = kChunk, NSL = L::NSL, RW = L::RW, RU = L::RU;
    constexpr int LK = L::LK, LV = L::LV, LC = L::LC, LKV = L::LKV;
    extern __shared__ float sm[];
    float *Kb = sm;                  // [CH][LKV]  k, then k e^g, then the X / O partials (stride LV)
    float *Qb = Kb + CH * LKV;       // [CH][LK]   q, then s q e^g
    float *Gb = Qb + CH * LK;        // [CH][LK]   log_alpha, then g, then W
    float *Kc = Gb + CH * LK;        // [CH][LK]   k e^{g_last - g}
    float *Vb = Kc + CH * LK;        // [CH][LV]   v, then u
    float *Ab = Vb + CH * LV;        // [CH][LC]   A, then T'
    float *Pb = Ab + CH * LC;        // [CH][LC]   P
    float *Tb = Pb + CH * LC;        // [CH][LC]   T (lower); partial products in the upper blocks
    float *bt = Tb + CH * LC;        // [CH]       beta
    float *dC = bt + CH;             // [DK]       e^{g_last}

    const int H = a.H;
    const int n = blockIdx.x / H, h = blockIdx.x % H;
    const int tid = threadIdx.x, j = tid % DV, sl = tid / DV;
    const Tin *qg = static_cast<const Tin *>(a.q);
    const Tin *kg = static_cast<const Tin *>(a.k);
    const Tin *vg = static_cast<const Tin *>(a.v);
    Tin *og = static_cast<Tin *>(a.out);
    const float scale = a.scale;

    int64_t t0, t1;
    kda::seq_bounds(a.cu_seqlens, n, a.T, a.T_total, t0, t1);

    float S[RW];
    const size_t sbase = (size_t)(n * H + h) * DK * DV;
#pragma unroll
    for (int i = 0; i < RW; ++i)
        S[i] = a.S0 ? a.S0[sbase + (size_t)(sl * RW + i) * DV + j] : 0.f;

    for (int64_t c0 = t0; c0 < t1; c0 += CH) {
        const int nr = (int)(t1 - c0 < (int64_t)CH ? t1 - c0 : (int64_t)CH);
        // 1. load the chunk (rows past the end of the sequence are zero).
        for (int idx = tid; idx < CH * DK; idx += kSimtThreads) {
            const int r = idx / DK, c = idx % DK;
            float kv = 0.f, qv = 0.f, lv = 0.f;
            if (r < nr) {
                const size_t off = ((size_t)(c0 + r) * H + h) * DK + c;
                kv = kda::to_f32(kg[off]);
                qv = kda::to_f32(qg[off]);
                lv = kda::gate_log_alpha<Tin>(a.gate_kind, a.gate, a.A_log, a.dt_bias,
                                              (size_t)(c0 + r) * H + h, h, c, DK);
            }
            Kb[r * LKV + c] = kv;
            Qb[r * LK + c] = qv;
            Gb[r * LK + c] = lv;
        }
        for (int idx = tid; idx < CH * DV; idx += kSimtThreads) {
            const int r = idx / DV, c = idx % DV;
            Vb[r * LV + c] = r < nr ? kda::to_f32(vg[((size_t)(c0 + r) * H + h) * DV + c]) : 0.f;
        }
        for (int r = tid; r < CH; r += kSimtThreads)
            bt[r] = r < nr ? kda::beta_of(a.beta[(size_t)(c0 + r) * H + h], a.flags) : 0.f;
        __syncthreads();

        // 2. unit-length keys / queries (KDA_NORM_K / KDA_NORM_Q), one warp per row, in place.
        if (a.flags & (kda::FLAG_NORM_K | kda::FLAG_NORM_Q)) {
            const int warp = tid >> 5, lane = tid & 31;
            for (int r = warp; r < CH; r += kSimtThreads / 32) {
                float kk = 0.f, qq = 0.f;
                for (int c = lane; c < DK; c += 32) {
                    kk = fmaf(Kb[r * LKV + c], Kb[r * LKV + c], kk);
                    qq = fmaf(Qb[r * LK + c], Qb[r * LK + c], qq);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    kk += __shfl_xor_sync(0xffffffffu, kk, o);
                    qq += __shfl_xor_sync(0xffffffffu, qq, o);
                }
                const float fk = (a.flags & kda::FLAG_NORM_K) ? 1.f / fmaxf(sqrtf(kk), 1e-12f) : 1.f;
                const float fq = (a.flags & kda::FLAG_NORM_Q) ? 1.f / fmaxf(sqrtf(qq), 1e-12f) : 1.f;
                for (int c = lane; c < DK; c += 32) {
                    Kb[r * LKV + c] *= fk;
                    Qb[r * LK + c] *= fq;
                }
            }
        }
        //    alpha = exp(log_alpha), in place.
        for (int idx = tid; idx < CH * DK; idx += kSimtThreads) {
            const int r = idx / DK, c = idx % DK;
            Gb[r * LK + c] = expf(Gb[r * LK + c]);
        }
        __syncthreads();

        // 3. A (strictly lower, times beta_r) and P (lower with diagonal, times s).
        //    Thread (i, cg) owns column i and channels c = 4 m + cg; it walks
        //    the rows r >= i carrying one running decay product per channel, and the
        //    four channel groups of a column are summed with warp shuffles.
        {
            constexpr int CPT = DK / 4;               // channels per thread
            const int i = tid >> 2, cg = tid & 3;
            float f[CPT];
#pragma unroll
            for (int m = 0; m < CPT; ++m) f[m] = 1.f;
            float ki[CPT];
#pragma unroll
            for (int m = 0; m < CPT; ++m) ki[m] = Kb[i * LKV + m * 4 + cg];
            for (int r = 0; r < CH; ++r) {
                float av = 0.f, pv = 0.f;
                if (r >= i) {
#pragma unroll
                    for (int m = 0; m < CPT; ++m) {
                        const int c = m * 4 + cg;
                        if (r > i) f[m] *= Gb[r * LK + c];
                        const float kd = ki[m] * f[m];
                        av = fmaf(Kb[r * LKV + c], kd, av);
                        pv = fmaf(Qb[r * LK + c], kd, pv);
                    }
                }
                av += __shfl_xor_sync(0xffffffffu, av, 1);
                pv += __shfl_xor_sync(0xffffffffu, pv, 1);
                av += __shfl_xor_sync(0xffffffffu, av, 2);
                pv += __shfl_xor_sync(0xffffffffu, pv, 2);
                if (cg == 0) {
                    Ab[r * LC + i] = i < r ? bt[r] * av : 0.f;
                    Pb[r * LC + i] = i <= r ? scale * pv : 0.f;
                }
            }
        }
        __syncthreads();

        // 4. decayed operands, one thread per channel: gamma (prefix products) for
        //    k gamma and s q gamma in place, kappa (suffix products) for K_C.
        for (int c = tid; c < DK; c += kSimtThreads) {
            float kap = 1.f;
            for (int r = CH - 1; r >= 0; --r) {
                Kc[r * LK + c] = Kb[r * LKV + c] * kap;
                kap *= Gb[r * LK + c];
            }
            float gam = 1.f;
            for (int r = 0; r < CH; ++r) {
                gam *= Gb[r * LK + c];
                Kb[r * LKV + c] *= gam;
                Qb[r * LK + c] *= scale * gam;
            }
            dC[c] = gam;
        }
        __syncthreads();

        // 5. T = (I + A)^{-1}, blocked: the four 16 x 16 diagonal blocks by forward
        //    substitution (warp w < 4 solves block w; lane i holds row i of the block of A and
        //    column i of T, row r of A is broadcast from lane r), then the blocks below by
        //    distance d = a - b: T_ab = -T_aa X_ab with X_ab = sum_{m=b}^{a-1} A_am T_mb, X_ab
        //    parked in the (unused) upper block (b, a) of Tb.
        {
            const int warp = tid >> 5, lane = tid & 31;
            if (warp < 4) {
                const int w = warp, i = lane & 15;
                const float *Abk = Ab + (16 * w) * LC + 16 * w;
                float arow[16], tcol[16];
#pragma unroll
                for (int m = 0; m < 16; ++m) arow[m] = Abk[i * LC + m];
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m < r; ++m) acc = fmaf(__shfl_sync(0xffffffffu, arow[m], r), tcol[m], acc);
                    tcol[r] = r < i ? 0.f : (r == i ? 1.f : -acc);
                }
                if (lane < 16) {
#pragma unroll
                    for (int r = 0; r < 16; ++r) Tb[(16 * w + r) * LC + 16 * w + i] = tcol[r];
                }
            }
            __syncthreads();
            for (int d = 1; d < 4; ++d) {
                const int nb = 4 - d;                       // blocks (b + d, b), b < nb
                for (int e = tid; e < nb * 256; e += kSimtThreads) {
                    const int b = e >> 8, r = (e >> 4) & 15, c = e & 15, ab = b + d;
                    float acc = 0.f;
                    for (int m = 16 * b; m < 16 * ab; ++m)
                        acc = fmaf(Ab[(16 * ab + r) * LC + m], Tb[m * LC + 16 * b + c], acc);
                    Tb[(16 * b + r) * LC + 16 * ab + c] = acc;      // X_ab, row r, column c
                }
                __syncthreads();
                for (int e = tid; e < nb * 256; e += kSimtThreads) {
                    const int b = e >> 8, r = (e >> 4) & 15, c = e & 15, ab = b + d;
                    float acc = 0.f;
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        acc = fmaf(Tb[(16 * ab + r) * LC + 16 * ab + k], Tb[(16 * b + k) * LC + 16 * ab + c], acc);
                    Tb[(16 * ab + r) * LC + 16 * b + c] = -acc;
                }
                __syncthreads();
            }
        }
        //    T' = T Diag(beta) (lower triangle of T, unit diagonal included).
        for (int p = tid; p < CH * CH; p += kSimtThreads) {
            const int r = p / CH, i = p % CH;
            Ab[r * LC + i] = i <= r ? Tb[r * LC + i] * bt[i] : 0.f;
        }
        __syncthreads();

        // 6. W = T' (k e^g) into Gb.   7. U = T' v for this thread's rows, column j.
        for (int idx = tid; idx < CH * DK; idx += kSimtThreads) {
            const int r = idx / DK, c = idx % DK;
            float w = 0.f;
            for (int i = 0; i <= r; ++i) w = fmaf(Ab[r * LC + i], Kb[i * LKV + c], w);
            Gb[r * LK + c] = w;
        }
        float u[RU];
#pragma unroll
        for (int m = 0; m < RU; ++m) {
            const int r = sl * RU + m;
            float acc = 0.f;
            for (int i = 0; i <= r; ++i) acc = fmaf(Ab[r * LC + i], Vb[i * LV + j], acc);
            u[m] = acc;
        }
        __syncthreads();

        // 8. X = W S (partials over this thread's state rows, summed slice by slice
        //    in a fixed order into Kb), then u = U - X, stored into Vb.
        for (int rb = 0; rb < CH; rb += 16) {
            float x[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < RW; ++i) acc = fmaf(Gb[(rb + m) * LK + sl * RW + i], S[i], acc);
                x[m] = acc;
            }
            for (int s2 = 0; s2 < NSL; ++s2) {
                if (sl == s2) {
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        Kb[(rb + m) * LV + j] = (s2 ? Kb[(rb + m) * LV + j] : 0.f) + x[m];
                }
                __syncthreads();
            }
        }
#pragma unroll
        for (int m = 0; m < RU; ++m) {
            const int r = sl * RU + m;
            u[m] -= Kb[r * LV + j];
            Vb[r * LV + j] = u[m];
        }
        __syncthreads();

        // 9. o = (s q e^g) S + P u.
        for (int rb = 0; rb < CH; rb += 16) {
            float x[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < RW; ++i) acc = fmaf(Qb[(rb + m) * LK + sl * RW + i], S[i], acc);
                x[m] = acc;
            }
            for (int s2 = 0; s2 < NSL; ++s2) {
                if (sl == s2) {
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        Kb[(rb + m) * LV + j] = (s2 ? Kb[(rb + m) * LV + j] : 0.f) + x[m];
                }
                __syncthreads();
            }
        }
#pragma unroll
        for (int m = 0; m < RU; ++m) {
            const int r = sl * RU + m;
            if (r < nr) {
                float acc = Kb[r * LV + j];
                for (int i = 0; i <= r; ++i) acc = fmaf(Pb[r * LC + i], Vb[i * LV + j], acc);
                og[((size_t)(c0 + r) * H + h) * DV + j] = kda::from_f32<Tin>(acc);
            }
        }

        // 10. S <- Diag(e^{g_last}) S + K_C^T u.
#pragma unroll
        for (int i = 0; i < RW; ++i) {
            const int c = sl * RW + i;
            float acc = dC[c] * S[i];
            for (int r = 0; r < CH; ++r) acc = fmaf(Kc[r * LK + c], Vb[r * LV + j], acc);
            S[i] = acc;
        }
        __syncthreads();
    }

    if (a.S_final) {
#pragma unroll
        for (int i = 0; i < RW; ++i) a.S_final[sbase + (size_t)(sl * RW + i) * DV + j] = S[i];
    }
}

template <typename Tin, int DK, int DV>
cudaError_t launch(const KdaChunkArgs &a, cudaStream_t st) {
    const size_t smem = SimtLayout<DK, DV>::bytes;
    cudaError_t e = cudaFuncSetAttribute(kda_chunk_simt_kernel<Tin, DK, DV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((int64_t)a.N * a.H);
    kda_chunk_simt_kernel<Tin, DK, DV><<<grid, kSimtThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <typename Tin, int DK>
cudaError_t pick_dv(const KdaChunkArgs &a, cudaStream_t st) {
    switch (a.dv) {
    case 32: return launch<Tin, DK, 32>(a, st);
    case 64: return launch<Tin, DK, 64>(a, st);
    case 128: return launch<Tin, DK, 128>(a, st);
    }
    return cudaErrorInvalidValue;
}

template <typename Tin>
cudaError_t pick_dk(const KdaChunkArgs &a, cudaStream_t st) {
    switch (a.dk) {
    case 32: return pick_dv<Tin, 32>(a, st);
    case 64: return pick_dv<Tin, 64>(a, st);
    case 128: return pick_dv<Tin, 128>(a, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kda_simt
