// k_rope.cu -- compressed-key pooling (prefill and decode ring), indexer
// query rotation, and the attention layer's RoPE helper.
//
// Pooling follows "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section
// "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely": four raw
// indexer keys are averaged in FP32, (optionally) normalised, rotated with the
// first token's position and stored as one BF16 compressed key; the raw keys
// of the unfinished block live in a four-slot ring per request.  The flozi.net
// guide ("How a token moves through the model", item 2) gives the reason for
// rotating after pooling: keys of different positions are not averaged at
// different rotary phases.
//
// Angles and rotations are evaluated in fp64 with explicitly rounded
// multiplies (no FMA contraction) so that the BF16/FP32 rounding of the
// result is decided by the exact rotated value.  These kernels move a few MB;
// they are HBM/latency bound and use 16-byte vector accesses.
#include "internal.h"

namespace qsa {

namespace {

// Rotated value of dim e given the (scaled) pair members; fp64, no contraction.
__device__ __forceinline__ double rope_dim(double xe, double xpartner, int e, int half, double c, double s) {
    return (e < half) ? __dsub_rn(__dmul_rn(xe, c), __dmul_rn(xpartner, s))
                      : __dadd_rn(__dmul_rn(xe, c), __dmul_rn(xpartner, s));
}

__device__ __forceinline__ void rope_cs(const Rope &r, double pos, int pair, double &c, double &s) {
    double ang = __dmul_rn(__ddiv_rn(pos, r.pos_scale), rope_inv_freq(r, pair));
    sincos(ang, &s, &c);
}

template <typename T> struct Vec16;   // 16 consecutive elements
template <> struct Vec16<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[16]) {
        const uint4 *q = reinterpret_cast<const uint4 *>(p);
        uint4 a = q[0], b = q[1];
        const __nv_bfloat16 *ea = reinterpret_cast<const __nv_bfloat16 *>(&a);
        const __nv_bfloat16 *eb = reinterpret_cast<const __nv_bfloat16 *>(&b);
#pragma unroll
        for (int i = 0; i < 8; ++i) { v[i] = __bfloat162float(ea[i]); v[8 + i] = __bfloat162float(eb[i]); }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const double (&v)[16]) {
        uint4 a, b;
        __nv_bfloat16 *ea = reinterpret_cast<__nv_bfloat16 *>(&a);
        __nv_bfloat16 *eb = reinterpret_cast<__nv_bfloat16 *>(&b);
#pragma unroll
        for (int i = 0; i < 8; ++i) { ea[i] = d2bf(v[i]); eb[i] = d2bf(v[8 + i]); }
        uint4 *q = reinterpret_cast<uint4 *>(p);
        q[0] = a;
        q[1] = b;
    }
};
template <> struct Vec16<float> {
    static __device__ __forceinline__ void load(const float *p, float (&v)[16]) {
        const float4 *q = reinterpret_cast<const float4 *>(p);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float4 x = q[i];
            v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
        }
    }
    static __device__ __forceinline__ void store(float *p, const double (&v)[16]) {
        float4 *q = reinterpret_cast<float4 *>(p);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            q[i] = make_float4((float)v[4 * i], (float)v[4 * i + 1], (float)v[4 * i + 2], (float)v[4 * i + 3]);
    }
};

// One compressed key per 8 threads; 32 keys per 256-thread CTA.  Thread j of
// a key handles dims [16j, 16j + 16).
// 16 rotated values -> 16 FP8 E4M3 bytes.
__device__ __forceinline__ void store16_e4m3(uint8_t *dst, const double (&v)[16]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        w[i] = (uint32_t)d2e4m3x2(v[4 * i], v[4 * i + 1]) | ((uint32_t)d2e4m3x2(v[4 * i + 2], v[4 * i + 3]) << 16);
    *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
}

// FP8: the compressed keys are stored as FP8 E4M3 (raw keys stay T).
template <typename T, bool FP8 = false>
__global__ void __launch_bounds__(256) pool_prefill_kernel(const T *__restrict__ k_raw, void *__restrict__ k_pool_v,
                                                           int64_t nblk, int64_t pos0, int64_t raw_stride,
                                                           int64_t pool_stride, Rope rope, int rmsnorm, Paging pg,
                                                           unsigned *status) {
    __shared__ float mean_s[32][kIdxDim];
    const int seq = blockIdx.y;
    const int kl = threadIdx.x >> 3;    // key within CTA
    const int j = threadIdx.x & 7;
    const int64_t blk = (int64_t)blockIdx.x * 32 + kl;
    const bool live = blk < nblk;
    float m[16];
    if (live) {
        const T *src = k_raw + ((int64_t)seq * raw_stride + blk * kBlock) * kIdxDim + 16 * j;
        float r0[16], r1[16], r2[16], r3[16];
        Vec16<T>::load(src, r0);
        Vec16<T>::load(src + kIdxDim, r1);
        Vec16<T>::load(src + 2 * kIdxDim, r2);
        Vec16<T>::load(src + 3 * kIdxDim, r3);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float s = __fadd_rn(r0[i], r1[i]);
            s = __fadd_rn(s, r2[i]);
            s = __fadd_rn(s, r3[i]);
            m[i] = __fmul_rn(s, 0.25f);
            mean_s[kl][16 * j + i] = m[i];
        }
    }
    double inv = 1.0;
    if (rmsnorm) {
        double ss = 0.0;
        if (live)
#pragma unroll
            for (int i = 0; i < 16; ++i) ss += (double)m[i] * (double)m[i];
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        ss += __shfl_xor_sync(0xffffffffu, ss, 4);
        inv = 1.0 / sqrt(ss / kIdxDim + 1e-6);
    }
    __syncwarp();
    if (!live) return;
    const int R = rope.rotary_dim, half = R >> 1;
    const double pos = (double)(pos0 + blk * kBlock);
    double out[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int e = 16 * j + i;
        double xe = rmsnorm ? __dmul_rn((double)m[i], inv) : (double)m[i];
        if (e < R) {
            const int pr = e < half ? e + half : e - half;
            double xp = (double)mean_s[kl][pr];
            if (rmsnorm) xp = __dmul_rn(xp, inv);
            double c, s;
            rope_cs(rope, pos, e < half ? e : e - half, c, s);
            out[i] = rope_dim(xe, xp, e, half, c, s);
        } else {
            out[i] = xe;
        }
    }
    int64_t row = (int64_t)seq * pool_stride + pos0 / kBlock + blk;
    if (pg.table) {   // paged: the row of the block's first token slot
        const int64_t slot = paged_slot(pg, seq, pos0 + blk * kBlock);
        if (slot < 0) {
            if (j == 0) flag(status, QSA_DEV_BAD_INDEX);
            return;
        }
        row = slot / kBlock;
    }
    if constexpr (FP8) {
        store16_e4m3(static_cast<uint8_t *>(k_pool_v) + row * kIdxDim + 16 * j, out);
    } else {
        T *dst = static_cast<T *>(k_pool_v) + row * kIdxDim + 16 * j;
        Vec16<T>::store(dst, out);
    }
}

// Decode: one CTA of 128 threads per sequence, thread e owns dim e.
template <typename T, bool FP8 = false>
__global__ void __launch_bounds__(128) pool_decode_kernel(const T *__restrict__ k_new, T *__restrict__ ring,
                                                          void *__restrict__ k_pool_v,
                                                          const int32_t *__restrict__ seq_len, int64_t pool_stride,
                                                          Rope rope, int rmsnorm, Paging pg, unsigned *status) {
    __shared__ double out_s[kIdxDim];
    __shared__ float mean_s[kIdxDim];
    __shared__ double red[4];
    pdl_wait();      // k_new and seq_len may come from the previous kernel
    pdl_trigger();   // the indexer may launch; it waits for this grid before reading k_pool
    const int seq = blockIdx.x;
    const int e = threadIdx.x;
    const int64_t s = seq_len[seq];
    if (s < 1) {
        if (e == 0) flag(status, QSA_DEV_BAD_LENGTH);
        return;
    }
    const int64_t p = s - 1;
    T *rg = ring + (int64_t)seq * kBlock * kIdxDim;
    const T knew = k_new[(int64_t)seq * kIdxDim + e];
    rg[(p % kBlock) * kIdxDim + e] = knew;
    if (s % kBlock != 0) return;
    const int64_t b = s / kBlock - 1;
    int64_t row = (int64_t)seq * pool_stride + b;
    if (pg.table) {   // paged: the row of the block's first token slot
        const int64_t slot = paged_slot(pg, seq, b * kBlock);
        if (slot < 0) {
            if (e == 0) flag(status, QSA_DEV_BAD_INDEX);
            return;
        }
        row = slot / kBlock;
    } else if (b >= pool_stride) {
        if (e == 0) flag(status, QSA_DEV_BAD_LENGTH);
        return;
    }
    // slot 3 is the new key; slots 0..2 were written by earlier steps
    float r0 = to_float(rg[e]), r1 = to_float(rg[kIdxDim + e]), r2 = to_float(rg[2 * kIdxDim + e]);
    float r3 = to_float(knew);
    float sum = __fadd_rn(r0, r1);
    sum = __fadd_rn(sum, r2);
    sum = __fadd_rn(sum, r3);
    const float m = __fmul_rn(sum, 0.25f);
    mean_s[e] = m;
    double inv = 1.0;
    if (rmsnorm) {
        double ss = (double)m * (double)m;
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if ((e & 31) == 0) red[e >> 5] = ss;
    }
    __syncthreads();
    if (rmsnorm) inv = 1.0 / sqrt((red[0] + red[1] + red[2] + red[3]) / kIdxDim + 1e-6);
    const int R = rope.rotary_dim, half = R >> 1;
    double xe = rmsnorm ? __dmul_rn((double)m, inv) : (double)m;
    double out = xe;
    if (e < R) {
        const int pr = e < half ? e + half : e - half;
        double xp = (double)mean_s[pr];
        if (rmsnorm) xp = __dmul_rn(xp, inv);
        double c, sn;
        rope_cs(rope, (double)(s - kBlock), e < half ? e : e - half, c, sn);
        out = rope_dim(xe, xp, e, half, c, sn);
    }
    if constexpr (FP8) {   // pairs of dims -> one 16-bit store
        out_s[e] = out;
        __syncthreads();
        if ((e & 1) == 0)
            reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(k_pool_v) + row * kIdxDim)[e >> 1] =
                d2e4m3x2(out_s[e], out_s[e + 1]);
    } else {
        static_cast<T *>(k_pool_v)[row * kIdxDim + e] = from_double<T>(out);
    }
}

// Attention-layer RoPE: one CTA per (sequence, row), thread i < R/2 turns
// pair (i, i + R/2) of every head.
template <typename T>
__global__ void rope_apply_kernel(T *__restrict__ x, int64_t n, int H, int d, int64_t pos0, Rope rope) {
    const int64_t row = blockIdx.x;   // over B * n
    const int i = threadIdx.x;
    const int half = rope.rotary_dim >> 1;
    if (i >= half) return;
    const int64_t r = row % n;
    double c, s;
    rope_cs(rope, (double)(pos0 + r), i, c, s);
    T *base = x + row * (int64_t)H * d;
    for (int h = 0; h < H; ++h) {
        T *p = base + (int64_t)h * d;
        double a = to_float(p[i]), b = to_float(p[i + half]);
        double o0 = __dsub_rn(__dmul_rn(a, c), __dmul_rn(b, s));
        double o1 = __dadd_rn(__dmul_rn(b, c), __dmul_rn(a, s));
        p[i] = from_double<T>(o0);
        p[i + half] = from_double<T>(o1);
    }
}

// Indexer queries: one CTA of 128 threads per (sequence, query row), thread e
// owns dim e of all 4 heads.  mode 0: hi/lo bf16 planes of the FP32 head sum
// of the BF16-rounded rotated heads; mode 1: per-head bf16; mode 2: per-head fp32.
template <typename T>
__global__ void __launch_bounds__(128) rotate_index_q_kernel(const T *__restrict__ q_idx, int64_t n_q, int64_t q0,
                                                             Rope rope, int mode, void *out0, void *out1) {
    const int64_t row = blockIdx.x;   // over B * n_q
    const int e = threadIdx.x;
    const int64_t t = q0 + row % n_q;
    const int R = rope.rotary_dim, half = R >> 1;
    double c = 1.0, s = 0.0;
    int pr = e;
    if (e < R) {
        pr = e < half ? e + half : e - half;
        rope_cs(rope, (double)t, e < half ? e : e - half, c, s);
    }
    const T *src = q_idx + row * kIdxHeads * kIdxDim;
    float hsum = 0.0f;
#pragma unroll
    for (int h = 0; h < kIdxHeads; ++h) {
        double xe = to_float(src[h * kIdxDim + e]);
        double o = xe;
        if (e < R) o = rope_dim(xe, (double)to_float(src[h * kIdxDim + pr]), e, half, c, s);
        if (mode == 2) {
            reinterpret_cast<float *>(out0)[(row * kIdxHeads + h) * kIdxDim + e] = (float)o;
        } else {
            __nv_bfloat16 ob = d2bf(o);
            if (mode == 1)
                reinterpret_cast<__nv_bfloat16 *>(out0)[(row * kIdxHeads + h) * kIdxDim + e] = ob;
            else
                hsum = (h == 0) ? __bfloat162float(ob) : __fadd_rn(hsum, __bfloat162float(ob));
        }
    }
    if (mode == 0) {
        __nv_bfloat16 hi = __float2bfloat16_rn(hsum);
        __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(hsum, __bfloat162float(hi)));
        reinterpret_cast<__nv_bfloat16 *>(out0)[row * kIdxDim + e] = hi;
        reinterpret_cast<__nv_bfloat16 *>(out1)[row * kIdxDim + e] = lo;
    }
}

}  // namespace

cudaError_t launch_pool_prefill(const void *k_raw, void *k_pool, int B, int64_t nblk, int64_t pos0,
                                int64_t raw_stride, int64_t pool_stride, Rope rope, bool rmsnorm, bool bf16,
                                bool fp8, const Paging &pg, unsigned *status, cudaStream_t s) {
    if (nblk <= 0) return cudaSuccess;
    dim3 grid((unsigned)((nblk + 31) / 32), (unsigned)B);
    const int rn = rmsnorm ? 1 : 0;
    if (bf16 && fp8)
        pool_prefill_kernel<__nv_bfloat16, true><<<grid, 256, 0, s>>>(
            (const __nv_bfloat16 *)k_raw, k_pool, nblk, pos0, raw_stride, pool_stride, rope, rn, pg, status);
    else if (bf16)
        pool_prefill_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>((const __nv_bfloat16 *)k_raw, k_pool, nblk, pos0,
                                                                raw_stride, pool_stride, rope, rn, pg, status);
    else
        pool_prefill_kernel<float><<<grid, 256, 0, s>>>((const float *)k_raw, k_pool, nblk, pos0, raw_stride,
                                                        pool_stride, rope, rn, pg, status);
    return cudaGetLastError();
}

cudaError_t launch_pool_decode(const void *k_new, void *ring, void *k_pool, const int32_t *seq_len, int B,
                               int64_t pool_stride, Rope rope, bool rmsnorm, bool bf16, bool fp8, const Paging &pg,
                               unsigned *status, cudaStream_t s) {
    const int rn = rmsnorm ? 1 : 0;
    if (bf16 && fp8)
        return launch_pdl(pool_decode_kernel<__nv_bfloat16, true>, dim3(B), dim3(128), 0, s,
                          (const __nv_bfloat16 *)k_new, (__nv_bfloat16 *)ring, k_pool, seq_len, pool_stride, rope,
                          rn, pg, status);
    if (bf16)
        return launch_pdl(pool_decode_kernel<__nv_bfloat16, false>, dim3(B), dim3(128), 0, s,
                          (const __nv_bfloat16 *)k_new, (__nv_bfloat16 *)ring, k_pool, seq_len, pool_stride, rope,
                          rn, pg, status);
    return launch_pdl(pool_decode_kernel<float, false>, dim3(B), dim3(128), 0, s, (const float *)k_new, (float *)ring,
                      k_pool, seq_len, pool_stride, rope, rn, pg, status);
}

cudaError_t launch_rope_apply(void *x, int B, int64_t n, int H, int d, int64_t pos0, Rope rope, bool bf16,
                              cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    const int threads = ((rope.rotary_dim / 2) + 31) / 32 * 32;
    if (bf16)
        rope_apply_kernel<__nv_bfloat16><<<(unsigned)(B * n), threads, 0, s>>>((__nv_bfloat16 *)x, n, H, d, pos0,
                                                                               rope);
    else
        rope_apply_kernel<float><<<(unsigned)(B * n), threads, 0, s>>>((float *)x, n, H, d, pos0, rope);
    return cudaGetLastError();
}

cudaError_t launch_rotate_index_q(const void *q_idx, int B, int64_t n_q, int64_t q0, Rope rope, int mode,
                                  void *out0, void *out1, cudaStream_t s) {
    if (n_q <= 0) return cudaSuccess;
    const unsigned rows = (unsigned)(B * n_q);
    if (mode == 2)
        rotate_index_q_kernel<float><<<rows, 128, 0, s>>>((const float *)q_idx, n_q, q0, rope, mode, out0, out1);
    else
        rotate_index_q_kernel<__nv_bfloat16><<<rows, 128, 0, s>>>((const __nv_bfloat16 *)q_idx, n_q, q0, rope,
                                                                  mode, out0, out1);
    return cudaGetLastError();
}

}  // namespace qsa
