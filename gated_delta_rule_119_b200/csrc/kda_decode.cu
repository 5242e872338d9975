// Decode: L new tokens for each of N sequences, states in an indexed pool.
//
// The recurrence applied token by token, per (sequence n, head h), fp32 throughout
// ("Ten questions" Q3-Q8; the token loop of "22,580" §6.1), from the pool slot
// idx = state_idx[n] (n without an index table):
//   S~ = Diag(alpha) S          alpha = exp(log_alpha)  (any gate form)     forget
//   r_k = S~^T k,  r_q = S~^T (s q)                     two lookups, one pass
//   u  = beta (v - r_k)                                                     correct
//   S  = S~ + k u^T                                                         write
//   o  = S^T (s q) = r_q + u (k . s q)                                      read
// With KDA_NORM_K / KDA_NORM_Q the unit-length key and query are f_k k and f_q q for the
// per-token scalars f = 1 / max(||x||_2, 1e-12): the lookups are scaled after the
// reductions, the write uses k (f_k u)^T, and k . s q becomes f_k f_q (k . s q).  Without
// them both factors are exactly 1 and the general kernel does the one-token kernel's
// arithmetic in the same order, so L tokens in one call give bit for bit the results of L
// calls of one token.
//
// Memory-bound: each state (dk x dv fp32) is read once before the first token and written
// once after the last, whatever L is; between tokens it stays in registers.  Three kernels:
// the one-token step with the per-channel gate and no flags, one token of any other form, and
// L tokens.  One CTA of 256 threads per (n, h).  Thread (rg, cg) holds the float4 column group
// cg of the rows rg * ROWS .. rg * ROWS + ROWS - 1; a warp therefore reads whole 512-byte rows,
// so every load and store of the state is a fully coalesced 128-bit access.
#include "kda_common.cuh"

// Bit 1: a sequence's state index was >= the pool size (the sequence was skipped).
__device__ unsigned int g_kda_decode_status = 0;

namespace {

constexpr int kDecodeThreads = 256;

// The per-row arithmetic of both step kernels, on packed fp32 pairs (fma.rn.f32x2 and
// mul.rn.f32x2 round each lane exactly as fmaf and a plain product do; one instruction does
// two lanes).  A thread holds ROWS consecutive state rows (a warp reads ROWS whole rows), so the
// row scalars (alpha, k, s q) come from shared memory four at a time.

// Row s of the state decayed in place by al, and its share of the lookups r_k, r_q.
__device__ __forceinline__ void decay_lookup(float4 &s, float al, float k, float q, float4 &rk, float4 &rq) {
    const float2 a2 = make_float2(al, al), k2 = make_float2(k, k), q2 = make_float2(q, q);
    const float2 lo = __fmul2_rn(make_float2(s.x, s.y), a2), hi = __fmul2_rn(make_float2(s.z, s.w), a2);
    s = make_float4(lo.x, lo.y, hi.x, hi.y);
    const float2 klo = __ffma2_rn(k2, lo, make_float2(rk.x, rk.y)), khi = __ffma2_rn(k2, hi, make_float2(rk.z, rk.w));
    const float2 qlo = __ffma2_rn(q2, lo, make_float2(rq.x, rq.y)), qhi = __ffma2_rn(q2, hi, make_float2(rq.z, rq.w));
    rk = make_float4(klo.x, klo.y, khi.x, khi.y);
    rq = make_float4(qlo.x, qlo.y, qhi.x, qhi.y);
}

// The write of row s: s + k u.
__device__ __forceinline__ float4 write_row(float4 s, float k, float4 u) {
    const float2 k2 = make_float2(k, k);
    const float2 lo = __ffma2_rn(k2, make_float2(u.x, u.y), make_float2(s.x, s.y));
    const float2 hi = __ffma2_rn(k2, make_float2(u.z, u.w), make_float2(s.z, s.w));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
    const float2 lo = __fadd2_rn(make_float2(a.x, a.y), make_float2(b.x, b.y));
    const float2 hi = __fadd2_rn(make_float2(a.z, a.w), make_float2(b.z, b.w));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// V consecutive row scalars from shared memory (V = 4: one 16-byte load).
template <int V>
__device__ __forceinline__ void rows_of(const float *p, float *out) {
    if constexpr (V == 4) {
        const float4 x = *reinterpret_cast<const float4 *>(p);
        out[0] = x.x; out[1] = x.y; out[2] = x.z; out[3] = x.w;
    } else {
#pragma unroll
        for (int j = 0; j < V; ++j) out[j] = p[j];
    }
}

// Decay the thread's rows r0 .. r0 + ROWS - 1 and form their shares of r_k and r_q.
template <int ROWS>
__device__ __forceinline__ void decay_lookup_rows(float4 *s, const float *sa, const float *sk, const float *sq,
                                                  int r0, float4 &rk, float4 &rq) {
    constexpr int V = ROWS % 4 == 0 ? 4 : 1;
#pragma unroll
    for (int i = 0; i < ROWS; i += V) {
        float av[V], kv[V], qv[V];
        rows_of<V>(sa + r0 + i, av);
        rows_of<V>(sk + r0 + i, kv);
        rows_of<V>(sq + r0 + i, qv);
#pragma unroll
        for (int j = 0; j < V; ++j) decay_lookup(s[i + j], av[j], kv[j], qv[j], rk, rq);
    }
}

// The common step -- one token per sequence, the per-channel gate, no flags -- in its own
// kernel: the state loads are issued first, s q is formed as it is loaded, and the updated
// state is stored as soon as u is known.
template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kDecodeThreads) kda_decode_step_kernel(KdaDecodeArgs a) {
    constexpr int CG = DV / 4, RG = kDecodeThreads / CG, ROWS = DK / RG;
    static_assert(kDecodeThreads % CG == 0 && DK % RG == 0, "decode tiling");
    __shared__ __align__(16) float s_k[DK], s_q[DK], s_a[DK], s_v[DV];
    __shared__ float4 s_red[2][RG][CG];
    __shared__ float s_kq;

    const int pair = blockIdx.x;               // n * H + h
    const int H = a.H, n = pair / H, h = pair % H;
    const int idx = a.state_idx ? a.state_idx[n] : n;
    if (idx < 0) return;                       // padding: nothing read or written
    if (idx >= a.P) {
        if (threadIdx.x == 0) atomicOr(&g_kda_decode_status, 1u);
        return;
    }
    const int tid = threadIdx.x;
    const int cg = tid % CG, rg = tid / CG;
    float4 *S4 = reinterpret_cast<float4 *>(a.S + ((size_t)idx * H + h) * DK * DV);
    float4 s[ROWS];
#pragma unroll
    for (int i = 0; i < ROWS; ++i) s[i] = __ldcs(&S4[(size_t)(rg * ROWS + i) * CG + cg]);

    const Tin *qp = static_cast<const Tin *>(a.q) + (size_t)pair * DK;
    const Tin *kp = static_cast<const Tin *>(a.k) + (size_t)pair * DK;
    const Tin *vp = static_cast<const Tin *>(a.v) + (size_t)pair * DV;
    const float *lap = static_cast<const float *>(a.gate) + (size_t)pair * DK;
    for (int c = tid; c < DK; c += kDecodeThreads) {
        s_k[c] = kda::to_f32(kp[c]);
        s_q[c] = a.scale * kda::to_f32(qp[c]);
        s_a[c] = expf(lap[c]);
    }
    for (int j = tid; j < DV; j += kDecodeThreads) s_v[j] = kda::to_f32(vp[j]);
    __syncthreads();

    if (tid < 32) {                            // k . (s q), one warp
        float acc = 0.f;
        for (int c = tid; c < DK; c += 32) acc = fmaf(s_k[c], s_q[c], acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (tid == 0) s_kq = acc;
    }
    float4 rk = make_float4(0.f, 0.f, 0.f, 0.f), rq = rk;
    decay_lookup_rows<ROWS>(s, s_a, s_k, s_q, rg * ROWS, rk, rq);
    s_red[0][rg][cg] = rk;
    s_red[1][rg][cg] = rq;
    __syncthreads();

    float4 tk = make_float4(0.f, 0.f, 0.f, 0.f), tq = tk;
#pragma unroll 8
    for (int g = 0; g < RG; ++g) {
        tk = add4(tk, s_red[0][g][cg]);
        tq = add4(tq, s_red[1][g][cg]);
    }
    const float b = a.beta[pair];
    float4 u;
    u.x = b * (s_v[4 * cg + 0] - tk.x);
    u.y = b * (s_v[4 * cg + 1] - tk.y);
    u.z = b * (s_v[4 * cg + 2] - tk.z);
    u.w = b * (s_v[4 * cg + 3] - tk.w);
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
        const int r = rg * ROWS + i;
        __stcs(&S4[(size_t)r * CG + cg], write_row(s[i], s_k[r], u));
    }
    if (rg == 0) {
        const float kq = s_kq;
        Tin *op = static_cast<Tin *>(a.out) + (size_t)pair * DV + 4 * cg;
        op[0] = kda::from_f32<Tin>(fmaf(u.x, kq, tq.x));
        op[1] = kda::from_f32<Tin>(fmaf(u.y, kq, tq.y));
        op[2] = kda::from_f32<Tin>(fmaf(u.z, kq, tq.z));
        op[3] = kda::from_f32<Tin>(fmaf(u.w, kq, tq.w));
    }
}

// Any step: L tokens per sequence, every gate form, flags.  The tokens' inputs are staged in
// shared memory LB at a time, in one pass issued right after the state loads, and the
// per-token scalars (k . s q and the norm factors) of a batch are formed by one warp per
// token, so the token loop itself reads no global memory.  The reduction scratch alternates
// between two buffers from token to token: one barrier per token.
template <typename Tin, int DK, int DV, int LB>
__device__ __forceinline__ void decode_tokens(const KdaDecodeArgs &a) {
    constexpr int CG = DV / 4;                 // float4 column groups per state row
    constexpr int RG = kDecodeThreads / CG;    // row groups
    constexpr int ROWS = DK / RG;              // state rows per thread
    static_assert(kDecodeThreads % CG == 0 && DK % RG == 0, "decode tiling");
    static_assert(LB <= kDecodeThreads / 32, "one warp per staged token");

    __shared__ __align__(16) float s_k[LB][DK], s_q[LB][DK], s_a[LB][DK], s_v[LB][DV];
    __shared__ float4 s_red[2][2][RG][CG];
    __shared__ float s_fk[LB], s_fq[LB], s_kq[LB], s_b[LB];

    const int H = a.H;
    const int n = blockIdx.x / H, h = blockIdx.x % H;
    const int idx = a.state_idx ? a.state_idx[n] : n;
    if (idx < 0) return;                       // padding: nothing read or written
    if (idx >= a.P) {
        if (threadIdx.x == 0) atomicOr(&g_kda_decode_status, 1u);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int cg = tid % CG, rg = tid / CG;
    float4 *S4 = reinterpret_cast<float4 *>(a.S + ((size_t)idx * H + h) * DK * DV);

    // The state is the traffic that matters: issue all of this thread's loads first.
    float4 s[ROWS];
#pragma unroll
    for (int i = 0; i < ROWS; ++i) s[i] = __ldcs(&S4[(size_t)(rg * ROWS + i) * CG + cg]);

    const Tin *qg = static_cast<const Tin *>(a.q);
    const Tin *kg = static_cast<const Tin *>(a.k);
    const Tin *vg = static_cast<const Tin *>(a.v);
    Tin *og = static_cast<Tin *>(a.out);
    const int L = a.L, flags = a.flags, gate_kind = a.gate_kind;
    const bool norm_k = flags & kda::FLAG_NORM_K, norm_q = flags & kda::FLAG_NORM_Q;

    for (int l0 = 0; l0 < L; l0 += LB) {
        const int nb = L - l0 < LB ? L - l0 : LB;
        if (l0 > 0) __syncthreads();           // the previous batch is no longer read
        for (int e = tid; e < nb * DK; e += kDecodeThreads) {
            const int l = e / DK, c = e - l * DK;
            const size_t th = ((size_t)n * L + l0 + l) * H + h;
            s_k[l][c] = kda::to_f32(kg[th * DK + c]);
            s_q[l][c] = a.scale * kda::to_f32(qg[th * DK + c]);
            s_a[l][c] = expf(kda::gate_log_alpha<Tin>(gate_kind, a.gate, a.A_log, a.dt_bias, th, h, c, DK));
        }
        for (int e = tid; e < nb * DV; e += kDecodeThreads) {
            const int l = e / DV, j = e - l * DV;
            s_v[l][j] = kda::to_f32(vg[(((size_t)n * L + l0 + l) * H + h) * DV + j]);
        }
        if (tid < nb) s_b[tid] = kda::beta_of(a.beta[((size_t)n * L + l0 + tid) * H + h], flags);
        __syncthreads();

        if (warp < nb) {                       // k . q and, when asked for, the norms: one warp a token
            const int l = warp;
            float kq = 0.f, kk = 0.f, qq = 0.f;
            for (int c = lane; c < DK; c += 32) kq = fmaf(s_k[l][c], s_q[l][c], kq);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o);
            if (norm_k || norm_q) {
                for (int c = lane; c < DK; c += 32) {
                    kk = fmaf(s_k[l][c], s_k[l][c], kk);
                    qq = fmaf(s_q[l][c], s_q[l][c], qq);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    kk += __shfl_xor_sync(0xffffffffu, kk, o);
                    qq += __shfl_xor_sync(0xffffffffu, qq, o);
                }
            }
            if (lane == 0) {
                // s_q holds s q, so 1 / max(||q||, eps) = s / max(||s q||, s eps)
                const float fk = norm_k ? 1.f / fmaxf(sqrtf(kk), 1e-12f) : 1.f;
                const float fq = norm_q ? a.scale / fmaxf(sqrtf(qq), a.scale * 1e-12f) : 1.f;
                s_fk[l] = fk;
                s_fq[l] = fq;
                s_kq[l] = fk * fq * kq;
            }
        }

        for (int l = 0; l < nb; ++l) {
            const size_t th = ((size_t)n * L + l0 + l) * H + h;   // token-head row
            const int par = l & 1;
            float4 rk = make_float4(0.f, 0.f, 0.f, 0.f), rq = rk;
            decay_lookup_rows<ROWS>(s, s_a[l], s_k[l], s_q[l], rg * ROWS, rk, rq);
            s_red[par][0][rg][cg] = rk;
            s_red[par][1][rg][cg] = rq;
            __syncthreads();                   // also publishes the batch's per-token scalars

            float4 tk = make_float4(0.f, 0.f, 0.f, 0.f), tq = tk;
#pragma unroll 8
            for (int g = 0; g < RG; ++g) {
                tk = add4(tk, s_red[par][0][g][cg]);
                tq = add4(tq, s_red[par][1][g][cg]);
            }
            const float fk = s_fk[l], fq = s_fq[l];
            const float b = s_b[l];
            const float *vv = s_v[l];
            float4 u;
            u.x = b * (vv[4 * cg + 0] - fk * tk.x);
            u.y = b * (vv[4 * cg + 1] - fk * tk.y);
            u.z = b * (vv[4 * cg + 2] - fk * tk.z);
            u.w = b * (vv[4 * cg + 3] - fk * tk.w);
            const float4 uk = make_float4(fk * u.x, fk * u.y, fk * u.z, fk * u.w);
#pragma unroll
            for (int i = 0; i < ROWS; ++i) s[i] = write_row(s[i], s_k[l][rg * ROWS + i], uk);
            if (rg == 0) {
                const float kq = s_kq[l];
                Tin *op = og + th * DV + 4 * cg;
                op[0] = kda::from_f32<Tin>(fmaf(u.x, kq, fq * tq.x));
                op[1] = kda::from_f32<Tin>(fmaf(u.y, kq, fq * tq.y));
                op[2] = kda::from_f32<Tin>(fmaf(u.z, kq, fq * tq.z));
                op[3] = kda::from_f32<Tin>(fmaf(u.w, kq, fq * tq.w));
            }
        }
    }
#pragma unroll
    for (int i = 0; i < ROWS; ++i) __stcs(&S4[(size_t)(rg * ROWS + i) * CG + cg], s[i]);
}

// L tokens, staged four at a time.
template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kDecodeThreads) kda_decode_kernel(KdaDecodeArgs a) {
    decode_tokens<Tin, DK, DV, 4>(a);
}

// One token with a gate form or flags the step kernel does not take: three CTAs per SM (a few
// registers spill), so one CTA's state loads overlap another's arithmetic.
template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kDecodeThreads, 3) kda_decode_single_kernel(KdaDecodeArgs a) {
    decode_tokens<Tin, DK, DV, 1>(a);
}

template <typename Tin, int DK, int DV>
cudaError_t launch(const KdaDecodeArgs &a, cudaStream_t st) {
    const unsigned grid = (unsigned)((int64_t)a.N * a.H);
    if (a.L == 1 && a.gate_kind == kda::GATE_CHANNEL && a.flags == 0)
        kda_decode_step_kernel<Tin, DK, DV><<<grid, kDecodeThreads, 0, st>>>(a);
    else if (a.L == 1)
        kda_decode_single_kernel<Tin, DK, DV><<<grid, kDecodeThreads, 0, st>>>(a);
    else
        kda_decode_kernel<Tin, DK, DV><<<grid, kDecodeThreads, 0, st>>>(a);
    return cudaGetLastError();
}

template <typename Tin, int DK>
cudaError_t pick_dv(const KdaDecodeArgs &a, cudaStream_t st) {
    switch (a.dv) {
    case 32: return launch<Tin, DK, 32>(a, st);
    case 64: return launch<Tin, DK, 64>(a, st);
    case 128: return launch<Tin, DK, 128>(a, st);
    }
    return cudaErrorInvalidValue;
}

template <typename Tin>
cudaError_t pick_dk(const KdaDecodeArgs &a, cudaStream_t st) {
    switch (a.dk) {
    case 32: return pick_dv<Tin, 32>(a, st);
    case 64: return pick_dv<Tin, 64>(a, st);
    case 128: return pick_dv<Tin, 128>(a, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t kda_launch_decode(const KdaDecodeArgs &a, int dtype, cudaStream_t stream) {
    return dtype == 0 ? pick_dk<float>(a, stream) : pick_dk<__nv_bfloat16>(a, stream);
}

cudaError_t kda_decode_read_status(unsigned int *status, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(status, g_kda_decode_status, sizeof(unsigned int));
    if (e != cudaSuccess || !clear || *status == 0) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_kda_decode_status, &zero, sizeof(unsigned int));
}
