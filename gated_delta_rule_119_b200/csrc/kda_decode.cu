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
// once after the last, whatever L is; between tokens it stays in registers.  One CTA of 256
// threads per (n, h).  Thread (rg, cg) holds the float4 column group cg of rows rg, rg + RG,
// ...; a warp therefore reads whole 512-byte rows, so every load and store of the state is
// a fully coalesced 128-bit access.
#include "kda_common.cuh"

// Bit 1: a sequence's state index was >= the pool size (the sequence was skipped).
__device__ unsigned int g_kda_decode_status = 0;

namespace {

constexpr int kDecodeThreads = 256;

__device__ __forceinline__ float4 fma4(float s, float4 a, float4 acc) {
    acc.x = fmaf(s, a.x, acc.x);
    acc.y = fmaf(s, a.y, acc.y);
    acc.z = fmaf(s, a.z, acc.z);
    acc.w = fmaf(s, a.w, acc.w);
    return acc;
}

// The common step -- one token per sequence, the per-channel gate, no flags -- in its own
// kernel: the state loads are issued first, s q is formed as it is loaded, and the updated
// state is stored as soon as u is known.
template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kDecodeThreads) kda_decode_step_kernel(KdaDecodeArgs a) {
    constexpr int CG = DV / 4, RG = kDecodeThreads / CG, ROWS = DK / RG;
    static_assert(kDecodeThreads % CG == 0 && DK % RG == 0, "decode tiling");
    __shared__ float s_k[DK], s_q[DK], s_a[DK], s_v[DV];
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
    for (int i = 0; i < ROWS; ++i) s[i] = __ldcs(&S4[(size_t)(rg + i * RG) * CG + cg]);

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
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
        const int r = rg + i * RG;
        const float al = s_a[r];
        s[i].x *= al;
        s[i].y *= al;
        s[i].z *= al;
        s[i].w *= al;
        rk = fma4(s_k[r], s[i], rk);
        rq = fma4(s_q[r], s[i], rq);
    }
    s_red[0][rg][cg] = rk;
    s_red[1][rg][cg] = rq;
    __syncthreads();

    float4 tk = make_float4(0.f, 0.f, 0.f, 0.f), tq = tk;
#pragma unroll 8
    for (int g = 0; g < RG; ++g) {
        const float4 x = s_red[0][g][cg], y = s_red[1][g][cg];
        tk.x += x.x; tk.y += x.y; tk.z += x.z; tk.w += x.w;
        tq.x += y.x; tq.y += y.y; tq.z += y.z; tq.w += y.w;
    }
    const float b = a.beta[pair];
    float4 u;
    u.x = b * (s_v[4 * cg + 0] - tk.x);
    u.y = b * (s_v[4 * cg + 1] - tk.y);
    u.z = b * (s_v[4 * cg + 2] - tk.z);
    u.w = b * (s_v[4 * cg + 3] - tk.w);
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
        const int r = rg + i * RG;
        __stcs(&S4[(size_t)r * CG + cg], fma4(s_k[r], u, s[i]));
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

// Any step: L tokens per sequence, every gate form, flags.
template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kDecodeThreads) kda_decode_kernel(KdaDecodeArgs a) {
    constexpr int CG = DV / 4;                 // float4 column groups per state row
    constexpr int RG = kDecodeThreads / CG;    // row groups
    constexpr int ROWS = DK / RG;              // state rows per thread
    static_assert(kDecodeThreads % CG == 0 && DK % RG == 0, "decode tiling");

    __shared__ float s_k[DK], s_q[DK], s_a[DK], s_v[DV];
    __shared__ float4 s_red[2][RG][CG];
    __shared__ float s_fk, s_fq, s_kq;

    const int H = a.H;
    const int n = blockIdx.x / H, h = blockIdx.x % H;
    const int idx = a.state_idx ? a.state_idx[n] : n;
    if (idx < 0) return;                       // padding: nothing read or written
    if (idx >= a.P) {
        if (threadIdx.x == 0) atomicOr(&g_kda_decode_status, 1u);
        return;
    }
    const int tid = threadIdx.x;
    const int cg = tid % CG, rg = tid / CG;
    float4 *S4 = reinterpret_cast<float4 *>(a.S + ((size_t)idx * H + h) * DK * DV);

    // The state is the traffic that matters: issue all of this thread's loads first.
    float4 s[ROWS];
#pragma unroll
    for (int i = 0; i < ROWS; ++i) s[i] = __ldcs(&S4[(size_t)(rg + i * RG) * CG + cg]);

    const Tin *qg = static_cast<const Tin *>(a.q);
    const Tin *kg = static_cast<const Tin *>(a.k);
    const Tin *vg = static_cast<const Tin *>(a.v);
    Tin *og = static_cast<Tin *>(a.out);
    const int L = a.L, flags = a.flags, gate_kind = a.gate_kind;
    const bool norm_k = flags & kda::FLAG_NORM_K, norm_q = flags & kda::FLAG_NORM_Q;

    for (int l = 0; l < L; ++l) {
        const size_t th = ((size_t)n * L + l) * H + h;        // token-head row
        for (int c = tid; c < DK; c += kDecodeThreads) {
            s_k[c] = kda::to_f32(kg[th * DK + c]);
            s_q[c] = a.scale * kda::to_f32(qg[th * DK + c]);
            s_a[c] = expf(kda::gate_log_alpha<Tin>(gate_kind, a.gate, a.A_log, a.dt_bias, th, h, c, DK));
        }
        for (int j = tid; j < DV; j += kDecodeThreads) s_v[j] = kda::to_f32(vg[th * DV + j]);
        __syncthreads();

        if (tid < 32) {                        // k . q and, when asked for, the norms: one warp
            float kq = 0.f, kk = 0.f, qq = 0.f;
            for (int c = tid; c < DK; c += 32) kq = fmaf(s_k[c], s_q[c], kq);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, o);
            if (norm_k || norm_q) {
                for (int c = tid; c < DK; c += 32) {
                    kk = fmaf(s_k[c], s_k[c], kk);
                    qq = fmaf(s_q[c], s_q[c], qq);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    kk += __shfl_xor_sync(0xffffffffu, kk, o);
                    qq += __shfl_xor_sync(0xffffffffu, qq, o);
                }
            }
            if (tid == 0) {
                // s_q holds s q, so 1 / max(||q||, eps) = s / max(||s q||, s eps)
                const float fk = norm_k ? 1.f / fmaxf(sqrtf(kk), 1e-12f) : 1.f;
                const float fq = norm_q ? a.scale / fmaxf(sqrtf(qq), a.scale * 1e-12f) : 1.f;
                s_fk = fk;
                s_fq = fq;
                s_kq = fk * fq * kq;
            }
        }

        float4 rk = make_float4(0.f, 0.f, 0.f, 0.f), rq = rk;
#pragma unroll
        for (int i = 0; i < ROWS; ++i) {
            const int r = rg + i * RG;
            const float al = s_a[r];
            s[i].x *= al;
            s[i].y *= al;
            s[i].z *= al;
            s[i].w *= al;
            rk = fma4(s_k[r], s[i], rk);
            rq = fma4(s_q[r], s[i], rq);
        }
        s_red[0][rg][cg] = rk;
        s_red[1][rg][cg] = rq;
        __syncthreads();

        float4 tk = make_float4(0.f, 0.f, 0.f, 0.f), tq = tk;
#pragma unroll 8
        for (int g = 0; g < RG; ++g) {
            const float4 x = s_red[0][g][cg], y = s_red[1][g][cg];
            tk.x += x.x; tk.y += x.y; tk.z += x.z; tk.w += x.w;
            tq.x += y.x; tq.y += y.y; tq.z += y.z; tq.w += y.w;
        }
        const float fk = s_fk, fq = s_fq;
        const float b = kda::beta_of(a.beta[th], flags);
        float4 u;
        u.x = b * (s_v[4 * cg + 0] - fk * tk.x);
        u.y = b * (s_v[4 * cg + 1] - fk * tk.y);
        u.z = b * (s_v[4 * cg + 2] - fk * tk.z);
        u.w = b * (s_v[4 * cg + 3] - fk * tk.w);
        const float4 uk = make_float4(fk * u.x, fk * u.y, fk * u.z, fk * u.w);
#pragma unroll
        for (int i = 0; i < ROWS; ++i) s[i] = fma4(s_k[rg + i * RG], uk, s[i]);
        if (rg == 0) {
            const float kq = s_kq;
            Tin *op = og + th * DV + 4 * cg;
            op[0] = kda::from_f32<Tin>(fmaf(u.x, kq, fq * tq.x));
            op[1] = kda::from_f32<Tin>(fmaf(u.y, kq, fq * tq.y));
            op[2] = kda::from_f32<Tin>(fmaf(u.z, kq, fq * tq.z));
            op[3] = kda::from_f32<Tin>(fmaf(u.w, kq, fq * tq.w));
        }
        if (l + 1 < L) __syncthreads();         // the next token's inputs reuse shared memory
    }
#pragma unroll
    for (int i = 0; i < ROWS; ++i) __stcs(&S4[(size_t)(rg + i * RG) * CG + cg], s[i]);
}

template <typename Tin, int DK, int DV>
cudaError_t launch(const KdaDecodeArgs &a, cudaStream_t st) {
    const unsigned grid = (unsigned)((int64_t)a.N * a.H);
    if (a.L == 1 && a.gate_kind == kda::GATE_CHANNEL && a.flags == 0)
        kda_decode_step_kernel<Tin, DK, DV><<<grid, kDecodeThreads, 0, st>>>(a);
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
