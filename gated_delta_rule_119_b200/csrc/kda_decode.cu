// Decode step: one new token for N independent (sequence, head) states.
//
// The recurrence applied once, per (n, h), fp32 throughout
// ("Ten questions" Q3-Q8; the token loop of "22,580" §6.1):
//   S~ = Diag(alpha) S          alpha = exp(log_alpha)           forget
//   r_k = S~^T k,  r_q = S~^T (s q)                              two lookups, one pass
//   u  = beta (v - r_k)                                          correct
//   S  = S~ + k u^T                                              write (stored back)
//   o  = S^T (s q) = r_q + u (k . s q)                           read
//
// Memory-bound: each state (dk x dv fp32) is read once and written once.  One
// CTA of 256 threads per (n, h).  Thread (rg, cg) holds the float4 column group
// cg of rows rg, rg + RG, ...; a warp therefore reads whole 512-byte rows, so
// every load and store of the state is a fully coalesced 128-bit access.
#include "kda_common.cuh"

namespace {

constexpr int kDecodeThreads = 256;

__device__ __forceinline__ float4 fma4(float s, float4 a, float4 acc) {
    acc.x = fmaf(s, a.x, acc.x);
    acc.y = fmaf(s, a.y, acc.y);
    acc.z = fmaf(s, a.z, acc.z);
    acc.w = fmaf(s, a.w, acc.w);
    return acc;
}

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kDecodeThreads) kda_decode_kernel(KdaDecodeArgs a) {
    constexpr int CG = DV / 4;                 // float4 column groups per state row
    constexpr int RG = kDecodeThreads / CG;    // row groups
    constexpr int ROWS = DK / RG;              // state rows per thread
    static_assert(kDecodeThreads % CG == 0 && DK % RG == 0, "decode tiling");

    __shared__ float s_k[DK], s_q[DK], s_a[DK], s_v[DV];
    __shared__ float4 s_red[2][RG][CG];
    __shared__ float s_kq;

    const int pair = blockIdx.x;               // n * H + h
    const int tid = threadIdx.x;
    const int cg = tid % CG, rg = tid / CG;
    float4 *S4 = reinterpret_cast<float4 *>(a.S + (size_t)pair * DK * DV);

    // The state is the traffic that matters: issue all of this thread's loads first.
    float4 s[ROWS];
#pragma unroll
    for (int i = 0; i < ROWS; ++i) s[i] = __ldcs(&S4[(size_t)(rg + i * RG) * CG + cg]);

    const Tin *qp = static_cast<const Tin *>(a.q) + (size_t)pair * DK;
    const Tin *kp = static_cast<const Tin *>(a.k) + (size_t)pair * DK;
    const Tin *vp = static_cast<const Tin *>(a.v) + (size_t)pair * DV;
    for (int c = tid; c < DK; c += kDecodeThreads) {
        s_k[c] = kda::to_f32(kp[c]);
        s_q[c] = a.scale * kda::to_f32(qp[c]);
        s_a[c] = expf(a.log_alpha[(size_t)pair * DK + c]);
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

template <typename Tin, int DK, int DV>
cudaError_t launch(const KdaDecodeArgs &a, cudaStream_t st) {
    const unsigned grid = (unsigned)((int64_t)a.N * a.H);
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
