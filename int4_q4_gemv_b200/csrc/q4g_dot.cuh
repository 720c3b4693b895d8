// The integer block dot product of the q4_0 GEMV kernels and its helpers.
#pragma once

#include "q4g_common.cuh"

namespace q4g {

// x digits of the integer dot product per block and activation row: 4 uint4
// (digit 0 / 1 of the low / high 16 columns), see block_dot_int.
constexpr int kDigitQuads = 4;

// Digits of 4 consecutive columns of one block (see block_dot_int):
// X_i = rint(x_i * 2^(29 - Emax)), |X_i| < 2^15 (the scaling is a power of two).
// Returns one packed word per digit (byte e = digit of column e: byte 0 of X
// unsigned, byte 1 signed) and adds the digit sums to sd.
Q4G_DEV void digits4(const __half (&h)[4], int em, uint32_t (&wd)[2], int (&sd)[2]) {
  const float sc = __int_as_float((29 - em + 127) << 23);
  // round to nearest even through the fp32 adder: x * sc is exact and
  // |x * sc| < 2^15, so x * sc + 1.5 * 2^23 rounds once at unit spacing and its
  // bit pattern minus that of 1.5 * 2^23 is the integer
  int X[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) X[e] = __float_as_int(fmaf(__half2float(h[e]), sc, 12582912.0f)) - 0x4B400000;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const uint32_t sel = 0x0040u | (uint32_t)(t * 0x11);  // bytes (x.b_t, y.b_t)
    const uint32_t lo = __byte_perm((uint32_t)X[0], (uint32_t)X[1], sel);
    const uint32_t hi = __byte_perm((uint32_t)X[2], (uint32_t)X[3], sel);
    wd[t] = __byte_perm(lo, hi, 0x5410);
  }
  sd[0] += dp4a_uu(wd[0], 0x01010101u, 0);
  int s1;
  asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(s1) : "r"(wd[1]), "r"(0x01010101u), "r"(0));
  sd[1] += s1;
}

Q4G_DEV int half_exp(__half h) {
  const int E = (__half_as_ushort(h) >> 10) & 31;
  return E ? E : 1;
}

// Digits of one whole 32-column block in one lane (see block_dot_int): xv[q]
// holds columns 8q .. 8q+7 as fp16. The largest exponent field comes from the
// largest magnitude (fp16 bit patterns of |x| order like the values; zero and
// subnormals count as exponent 1).
Q4G_DEV void lane_block_digits(const uint4 (&xv)[4], uint4 (&g)[kDigitQuads], int4& cv) {
  uint32_t mx = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    mx = __vmaxu2(mx, xv[q].x & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, xv[q].y & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, xv[q].z & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, xv[q].w & 0x7FFF7FFFu);
  }
  const uint32_t mh = max(mx & 0xFFFFu, mx >> 16);
  const int em = max((int)((mh >> 10) & 31u), 1);
  int sd[2] = {0, 0};
  uint32_t words[2][8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint32_t w0 = (&xv[q >> 1].x)[2 * (q & 1)], w1 = (&xv[q >> 1].x)[2 * (q & 1) + 1];
    const __half h4[4] = {__ushort_as_half((unsigned short)(w0 & 0xFFFFu)), __ushort_as_half((unsigned short)(w0 >> 16)),
                          __ushort_as_half((unsigned short)(w1 & 0xFFFFu)), __ushort_as_half((unsigned short)(w1 >> 16))};
    uint32_t wd[2];
    digits4(h4, em, wd, sd);
    words[0][q] = wd[0];
    words[1][q] = wd[1];
  }
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    g[2 * t] = make_uint4(words[t][0], words[t][1], words[t][2], words[t][3]);
    g[2 * t + 1] = make_uint4(words[t][4], words[t][5], words[t][6], words[t][7]);
  }
  cv = make_int4(-8 * sd[0], -8 * sd[1], 0, (em - 29 + 127) << 23);
}

// ---------------------------------------------------------------------------
// Integer form of the block dot product.
//
// x of one block (32 fp16 values) becomes signed 16-bit fixed point relative to
// the block's largest exponent: X_i = round(x_i * 2^(29 - Emax)), |X_i| < 2^15,
// exact for every value within 2^4 of the block maximum; the rest carry an
// error of at most 2^-15 of the block maximum. x_i ~= X_i * 2^(Emax - 29).
// The code byte b of a block holds column b in its low nibble and column b + 16
// in its high nibble, so a code word w gives the four low codes as
// w & 0x0F0F0F0F and the four high codes as (w >> 4) & 0x0F0F0F0F.
// X splits into bytes X = d0 + 256 d1 (d0 unsigned, d1 signed), and
//   sum_i (c_i - 8) X_i = S0 + 256 S1,  S_t = sum_i c_i d_t,i - 8 sum_i d_t,i,
// each S_t a chain of 4-way byte dot products (dp4a) started at the constant
// -8 sum_i d_t,i. S0, S1 and S0 + 256 S1 (|.| <= 32 * 8 * 2^15 = 2^23) are exact
// in int32 and the last one in fp32.
// Layout per x row j: dg[j][2t + h][blk] holds digit t of columns 16h..16h+15
// of block blk (16 bytes), bc[j][blk] = (-8 D0, -8 D1, 0, bits of 2^(Emax-29))
// with D_t = sum_i d_t,i, written by stage_digits.
// ---------------------------------------------------------------------------
Q4G_DEV float block_dot_int(const uint4 q, const uint4 (&g)[kDigitQuads], const int4 c) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  int s0 = c.x, s1 = c.y;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint32_t lo = w[t] & 0x0F0F0F0Fu, hi = (w[t] >> 4) & 0x0F0F0F0Fu;
    s0 = dp4a_uu(lo, (&g[0].x)[t], s0);
    s0 = dp4a_uu(hi, (&g[1].x)[t], s0);
    s1 = dp4a_us(lo, (&g[2].x)[t], s1);
    s1 = dp4a_us(hi, (&g[3].x)[t], s1);
  }
  return (float)(s1 * 256 + s0);
}

// Sum v[0..R) over the 32 lanes: after the butterfly, lanes with (lane & (32/R
// - 1)) == 0 hold the total of row cs_row<R>(lane).
template <int R>
Q4G_DEV float cs_reduce_rows(float (&v)[R], int lane) {
#pragma unroll
  for (int h = R / 2, o = 16; h >= 1; h >>= 1, o >>= 1) {
    const bool upper = lane & o;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = upper ? v[i] : v[i + h];
      const float keep = upper ? v[i + h] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  float t = v[0];
#pragma unroll
  for (int o = 16 / R; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  return t;
}
template <int R>
Q4G_DEV int cs_row(int lane) {
  int r = 0;
#pragma unroll
  for (int h = R / 2, o = 16; h >= 1; h >>= 1, o >>= 1) r += (lane & o) ? h : 0;
  return r;
}

}  // namespace q4g
