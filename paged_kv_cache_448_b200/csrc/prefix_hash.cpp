// prefix_hash.cpp — content hashes of full KV blocks for prefix caching.
//
// "大模型推理KV Cache内存管理与PagedAttention分页显存实战" (Prefix Caching):
// the KV blocks of a system prompt and of earlier turns are reused across
// requests, and shareable prefix blocks are recognised by hash matching. The
// page names no hash function. A block's identity here is the SHA-256
// (FIPS 180-4) of its parent block's 32-byte hash followed by the block's
// token ids as little-endian int32; the first block's parent is 32 zero
// bytes. Chaining makes equal hashes mean equal whole prefixes, and a
// 256-bit hash makes an accidental match (which would silently reuse another
// prompt's keys and values) practically impossible.
//
// SHA-256 follows the standard's description: 512-bit message blocks, the
// 64-entry message schedule, 64 compression rounds. Its round constants and
// initial value are derived at first use from their definition in the
// standard (fractional parts of the cube roots of the first 64 primes and of
// the square roots of the first 8), not typed in.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "paged.h"
#include "status.h"

namespace paged {
namespace {

struct Constants {
  uint32_t k[64];
  uint32_t h0[8];
};

uint32_t frac_bits(long double x) {
  const long double f = x - std::floor(x);
  return static_cast<uint32_t>(std::floor(std::ldexp(f, 32)));
}

const Constants& constants() {
  static Constants c;
  static std::once_flag once;
  std::call_once(once, [] {
    int primes[64];
    int n = 0;
    for (int p = 2; n < 64; ++p) {
      bool prime = true;
      for (int d = 2; d * d <= p; ++d)
        if (p % d == 0) {
          prime = false;
          break;
        }
      if (prime) primes[n++] = p;
    }
    for (int i = 0; i < 64; ++i) c.k[i] = frac_bits(std::cbrt(static_cast<long double>(primes[i])));
    for (int i = 0; i < 8; ++i) c.h0[i] = frac_bits(std::sqrt(static_cast<long double>(primes[i])));
  });
  return c;
}

inline uint32_t rotr(uint32_t x, int n) { return (x >> n) | (x << (32 - n)); }

}  // namespace

class Sha256 {
 public:
  Sha256() : c_(constants()) { std::memcpy(h_, c_.h0, sizeof(h_)); }

  void update(const uint8_t* p, size_t n) {
    bits_ += static_cast<uint64_t>(n) * 8;
    while (n > 0) {
      const size_t take = std::min(n, sizeof(buf_) - fill_);
      std::memcpy(buf_ + fill_, p, take);
      fill_ += take;
      p += take;
      n -= take;
      if (fill_ == sizeof(buf_)) {
        compress(buf_);
        fill_ = 0;
      }
    }
  }

  // Padding: a 1 bit, zeros up to 56 bytes mod 64, the message length in bits
  // as a big-endian 64-bit number.
  void finish(uint8_t out[32]) {
    const uint64_t bits = bits_;
    const uint8_t one = 0x80, zero = 0;
    update(&one, 1);
    while (fill_ != 56) update(&zero, 1);
    uint8_t len[8];
    for (int i = 0; i < 8; ++i) len[i] = static_cast<uint8_t>(bits >> (56 - 8 * i));
    update(len, 8);
    for (int i = 0; i < 8; ++i)
      for (int j = 0; j < 4; ++j) out[4 * i + j] = static_cast<uint8_t>(h_[i] >> (24 - 8 * j));
  }

 private:
  void compress(const uint8_t* blk) {
    uint32_t w[64];
    for (int t = 0; t < 16; ++t)
      w[t] = (uint32_t(blk[4 * t]) << 24) | (uint32_t(blk[4 * t + 1]) << 16) |
             (uint32_t(blk[4 * t + 2]) << 8) | uint32_t(blk[4 * t + 3]);
    for (int t = 16; t < 64; ++t) {
      const uint32_t s0 = rotr(w[t - 15], 7) ^ rotr(w[t - 15], 18) ^ (w[t - 15] >> 3);
      const uint32_t s1 = rotr(w[t - 2], 17) ^ rotr(w[t - 2], 19) ^ (w[t - 2] >> 10);
      w[t] = s1 + w[t - 7] + s0 + w[t - 16];
    }
    uint32_t a = h_[0], b = h_[1], c = h_[2], d = h_[3], e = h_[4], f = h_[5], g = h_[6],
             h = h_[7];
    for (int t = 0; t < 64; ++t) {
      const uint32_t S1 = rotr(e, 6) ^ rotr(e, 11) ^ rotr(e, 25);
      const uint32_t ch = (e & f) ^ (~e & g);
      const uint32_t t1 = h + S1 + ch + c_.k[t] + w[t];
      const uint32_t S0 = rotr(a, 2) ^ rotr(a, 13) ^ rotr(a, 22);
      const uint32_t maj = (a & b) ^ (a & c) ^ (b & c);
      const uint32_t t2 = S0 + maj;
      h = g;
      g = f;
      f = e;
      e = d + t1;
      d = c;
      c = b;
      b = a;
      a = t1 + t2;
    }
    h_[0] += a; h_[1] += b; h_[2] += c; h_[3] += d;
    h_[4] += e; h_[5] += f; h_[6] += g; h_[7] += h;
  }

  const Constants& c_;
  uint32_t h_[8];
  uint8_t buf_[64];
  size_t fill_ = 0;
  uint64_t bits_ = 0;
};

namespace {

void block_hash(const uint8_t* parent, const int32_t* tokens, int32_t n, uint8_t out[32]) {
  Sha256 s;
  uint8_t zeros[32] = {};
  s.update(parent ? parent : zeros, 32);
  for (int32_t i = 0; i < n; ++i) {
    const uint32_t t = static_cast<uint32_t>(tokens[i]);
    const uint8_t le[4] = {uint8_t(t), uint8_t(t >> 8), uint8_t(t >> 16), uint8_t(t >> 24)};
    s.update(le, 4);
  }
  s.finish(out);
}

}  // namespace
}  // namespace paged

using paged::clear_error;
using paged::fail;

extern "C" {

PA_API pa_status pa_sha256(const void* data, int64_t n, uint8_t out[32]) {
  clear_error();
  if (n < 0 || (n > 0 && !data) || !out) return fail(PA_ERR_INVALID_ARG, "sha256: bad args");
  paged::Sha256 s;
  s.update(static_cast<const uint8_t*>(data), static_cast<size_t>(n));
  s.finish(out);
  return PA_OK;
}

PA_API pa_status pa_block_hash(const uint8_t* parent, const int32_t* tokens, int32_t num_tokens,
                               uint8_t out[32]) {
  clear_error();
  if (num_tokens < 0 || (num_tokens > 0 && !tokens) || !out)
    return fail(PA_ERR_INVALID_ARG, "block_hash: bad args");
  paged::block_hash(parent, tokens, num_tokens, out);
  return PA_OK;
}

PA_API pa_status pa_prompt_block_hashes(const int32_t* tokens, int64_t num_tokens,
                                        int32_t block_size, uint8_t* hashes_out) {
  clear_error();
  if (num_tokens < 0 || block_size <= 0 || (num_tokens > 0 && !tokens))
    return fail(PA_ERR_INVALID_ARG, "prompt_block_hashes: bad args");
  const int64_t full = num_tokens / block_size;
  if (full > 0 && !hashes_out) return fail(PA_ERR_INVALID_ARG, "prompt_block_hashes: null output");
  for (int64_t j = 0; j < full; ++j)
    paged::block_hash(j == 0 ? nullptr : hashes_out + 32 * (j - 1), tokens + j * block_size,
                      block_size, hashes_out + 32 * j);
  return PA_OK;
}

}  // extern "C"
