// BLAKE2b (RFC 7693) with a 16-byte digest and no key: the cache key of a
// token prefix in the host prefix cache.  Written from the RFC's description:
// 64-bit words, 12 rounds of the G mixing function over a 16-word work
// vector, message schedule SIGMA, initialisation vector equal to SHA-512's,
// parameter block folded into h[0], a byte counter and a final-block flag.
// The state can be copied, so the digest of every prefix of a stream costs
// one finalisation each.
#pragma once

#include <cstdint>
#include <cstring>

namespace pkv {

class Blake2b128 {
 public:
  Blake2b128() {
    for (int i = 0; i < 8; ++i) h_[i] = kIV[i];
    h_[0] ^= 0x01010000ull ^ kOutBytes;  // depth 1, fanout 1, no key, digest length
  }

  void update(const uint8_t* p, size_t n) {
    while (n > 0) {
      if (fill_ == 128) {  // a full buffer is compressed only once more data arrives
        t_ += 128;
        compress(false);
        fill_ = 0;
      }
      const size_t k = n < 128 - fill_ ? n : 128 - fill_;
      std::memcpy(buf_ + fill_, p, k);
      fill_ += k;
      p += k;
      n -= k;
    }
  }

  // Digest of everything absorbed so far; the object itself is unchanged.
  void digest(uint8_t out[16]) const {
    Blake2b128 c = *this;
    c.t_ += c.fill_;
    std::memset(c.buf_ + c.fill_, 0, 128 - c.fill_);
    c.compress(true);
    for (int i = 0; i < 16; ++i) out[i] = static_cast<uint8_t>(c.h_[i / 8] >> (8 * (i % 8)));
  }

 private:
  static constexpr uint64_t kOutBytes = 16;
  static constexpr uint64_t kIV[8] = {0x6a09e667f3bcc908ull, 0xbb67ae8584caa73bull, 0x3c6ef372fe94f82bull,
                                      0xa54ff53a5f1d36f1ull, 0x510e527fade682d1ull, 0x9b05688c2b3e6c1full,
                                      0x1f83d9abfb41bd6bull, 0x5be0cd19137e2179ull};
  static constexpr uint8_t kSigma[10][16] = {
      {0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15}, {14, 10, 4, 8, 9, 15, 13, 6, 1, 12, 0, 2, 11, 7, 5, 3},
      {11, 8, 12, 0, 5, 2, 15, 13, 10, 14, 3, 6, 7, 1, 9, 4}, {7, 9, 3, 1, 13, 12, 11, 14, 2, 6, 5, 10, 4, 0, 15, 8},
      {9, 0, 5, 7, 2, 4, 10, 15, 14, 1, 11, 12, 6, 8, 3, 13}, {2, 12, 6, 10, 0, 11, 8, 3, 4, 13, 7, 5, 15, 14, 1, 9},
      {12, 5, 1, 15, 14, 13, 4, 10, 0, 7, 6, 3, 9, 2, 8, 11}, {13, 11, 7, 14, 12, 1, 3, 9, 5, 0, 15, 4, 8, 6, 2, 10},
      {6, 15, 14, 9, 11, 3, 0, 8, 12, 2, 13, 7, 1, 4, 10, 5}, {10, 2, 8, 4, 7, 6, 1, 5, 15, 11, 9, 14, 3, 12, 13, 0}};

  static uint64_t rotr(uint64_t x, int r) { return (x >> r) | (x << (64 - r)); }

  static void mix(uint64_t* v, int a, int b, int c, int d, uint64_t x, uint64_t y) {
    v[a] = v[a] + v[b] + x;
    v[d] = rotr(v[d] ^ v[a], 32);
    v[c] = v[c] + v[d];
    v[b] = rotr(v[b] ^ v[c], 24);
    v[a] = v[a] + v[b] + y;
    v[d] = rotr(v[d] ^ v[a], 16);
    v[c] = v[c] + v[d];
    v[b] = rotr(v[b] ^ v[c], 63);
  }

  void compress(bool last) {
    uint64_t m[16], v[16];
    for (int i = 0; i < 16; ++i) {
      uint64_t w = 0;
      for (int b = 7; b >= 0; --b) w = (w << 8) | buf_[8 * i + b];  // little-endian words
      m[i] = w;
    }
    for (int i = 0; i < 8; ++i) {
      v[i] = h_[i];
      v[i + 8] = kIV[i];
    }
    v[12] ^= t_;  // byte counter (inputs here stay far below 2^64 bytes)
    if (last) v[14] = ~v[14];
    for (int r = 0; r < 12; ++r) {
      const uint8_t* s = kSigma[r % 10];
      mix(v, 0, 4, 8, 12, m[s[0]], m[s[1]]);
      mix(v, 1, 5, 9, 13, m[s[2]], m[s[3]]);
      mix(v, 2, 6, 10, 14, m[s[4]], m[s[5]]);
      mix(v, 3, 7, 11, 15, m[s[6]], m[s[7]]);
      mix(v, 0, 5, 10, 15, m[s[8]], m[s[9]]);
      mix(v, 1, 6, 11, 12, m[s[10]], m[s[11]]);
      mix(v, 2, 7, 8, 13, m[s[12]], m[s[13]]);
      mix(v, 3, 4, 9, 14, m[s[14]], m[s[15]]);
    }
    for (int i = 0; i < 8; ++i) h_[i] ^= v[i] ^ v[i + 8];
  }

  uint64_t h_[8];
  uint64_t t_ = 0;
  uint8_t buf_[128] = {};
  size_t fill_ = 0;
};

// Appends token ids to a digest as little-endian int32.
inline void blake2b_tokens(Blake2b128* st, const int32_t* tokens, int n) {
  uint8_t b[64];
  while (n > 0) {
    const int k = n < 16 ? n : 16;
    for (int i = 0; i < k; ++i) {
      const uint32_t u = static_cast<uint32_t>(tokens[i]);
      b[4 * i] = static_cast<uint8_t>(u);
      b[4 * i + 1] = static_cast<uint8_t>(u >> 8);
      b[4 * i + 2] = static_cast<uint8_t>(u >> 16);
      b[4 * i + 3] = static_cast<uint8_t>(u >> 24);
    }
    st->update(b, static_cast<size_t>(4 * k));
    tokens += k;
    n -= k;
  }
}

}  // namespace pkv
