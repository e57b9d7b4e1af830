// Host build of the library's full-BPTT engine (bptt_core.h), for the CPU
// tests only: the same functors the CUDA kernels run, executed in a loop in
// fp64, so that their index arithmetic and the reverse-time schedule can be
// checked against the gradient oracle without a GPU, under
// AddressSanitizer.  The library never loads this program.
//
//   bptt_host names B S d H L W G F V tied merge_kind
//       prints "index name rows cols" for every stored tensor;
//   bptt_host run in.bin out.bin [passes]
//       in:  int32 B S d H L W G F V tied merge_kind seg; float64 alpha eps
//            rope_base; int32 tok[B*S]; float64 wts[B*(S-1)]; float64 of every
//            stored tensor in index order;
//       out: float64 logp[B*(S-1)], then the gradient of every stored tensor.
//       passes (default 1): run the pass that many times on one engine (the
//       way the library keeps it between calls); gradients accumulate.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "bptt_core.h"

using namespace rlt::bptt;

struct HostBackend {
  std::vector<void*> mem;
  ~HostBackend() {
    for (void* p : mem) free(p);
  }
  template <class T> T* alloc(size_t n) {
    T* p = static_cast<T*>(calloc(n ? n : 1, sizeof(T)));
    mem.push_back(p);
    return p;
  }
  template <class T> void zero(T* p, size_t n) { memset(p, 0, n * sizeof(T)); }
  template <class T> void copy(T* dst, const T* src, size_t n) { memmove(dst, src, n * sizeof(T)); }
  template <class T> void upload(T* dst, const T* src, size_t n) { memcpy(dst, src, n * sizeof(T)); }
  template <class K> void launch(const K& k, int64_t n) {
    for (int64_t i = 0; i < n; ++i) k(i);
  }
  int ok() const { return 0; }
  void range_push(const char*) {}
  void range_pop() {}
};

static bool read_all(FILE* f, void* p, size_t bytes) { return fread(p, 1, bytes, f) == bytes; }

int main(int argc, char** argv) {
  if (argc >= 13 && !strcmp(argv[1], "names")) {
    Dims D{};
    int v[11];
    for (int i = 0; i < 11; ++i) v[i] = atoi(argv[2 + i]);
    D.B = v[0]; D.S = v[1]; D.d = v[2]; D.H = v[3]; D.L = v[4]; D.W = v[5]; D.G = v[6]; D.F = v[7]; D.V = v[8];
    D.tied = v[9]; D.merge_kind = v[10];
    for (int i = 0; i < n_tensors(D); ++i) {
      if (!tensor_exists(D, i)) continue;
      int64_t r, c;
      tensor_shape(D, i, &r, &c);
      printf("%d %s %lld %lld\n", i, tensor_name(D, i).c_str(), (long long)r, (long long)c);
    }
    return 0;
  }
  if ((argc != 4 && argc != 5) || strcmp(argv[1], "run")) {
    fprintf(stderr, "usage: bptt_host names B S d H L W G F V tied merge_kind | run in.bin out.bin [passes]\n");
    return 2;
  }
  const int passes = argc == 5 ? atoi(argv[4]) : 1;
  if (passes < 1) return 2;
  FILE* f = fopen(argv[2], "rb");
  if (!f) return 3;
  int32_t h[12];
  double hf[3];
  if (!read_all(f, h, sizeof h) || !read_all(f, hf, sizeof hf)) return 4;
  Dims D{h[0], h[1], h[2], h[3], h[4], h[5], h[6], h[7], h[8], h[9], h[10], hf[0], hf[1], hf[2]};
  const int seg = h[11];
  if (D.B < 1 || D.S < 2 || D.d % D.H || (D.d / D.H) % 2 || D.d / D.H > kMaxHead) return 5;
  std::vector<int32_t> tok((size_t)D.B * D.S);
  std::vector<double> wts((size_t)D.B * (D.S - 1));
  if (!read_all(f, tok.data(), tok.size() * 4) || !read_all(f, wts.data(), wts.size() * 8)) return 4;
  const int n = n_tensors(D);
  std::vector<std::vector<double>> W(n), G(n);
  std::vector<const double*> wp(n, nullptr);
  std::vector<double*> gp(n, nullptr);
  for (int i = 0; i < n; ++i) {
    if (!tensor_exists(D, i)) continue;
    int64_t r, c;
    tensor_shape(D, i, &r, &c);
    W[i].resize((size_t)(r * c));
    G[i].assign((size_t)(r * c), 0.0);
    if (!read_all(f, W[i].data(), W[i].size() * 8)) return 4;
    wp[i] = W[i].data();
    gp[i] = G[i].data();
  }
  fclose(f);
  std::vector<double> logp(wts.size(), 0.0);
  HostBackend bk;
  Engine<HostBackend, double> eng(bk, D, wp.data(), gp.data());
  for (int p = 0; p < passes; ++p)
    if (eng.run(tok.data(), wts.data(), seg, logp.data()) != 0) return 6;
  FILE* o = fopen(argv[3], "wb");
  if (!o) return 3;
  fwrite(logp.data(), 8, logp.size(), o);
  for (int i = 0; i < n; ++i)
    if (!G[i].empty()) fwrite(G[i].data(), 8, G[i].size(), o);
  fclose(o);
  return 0;
}
