// C-ABI implementation of librace_attn.so: argument checks, planning, scratch
// layout and kernel launches.  The whole library is one translation unit so that the
// device status flag is a single __device__ symbol.
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "simt_kernels.cuh"
#include "tc_kernels.cuh"
#include "tc_ptx.cuh"
#include "tc_sweep.cuh"
#include "tc_sweep_pipe.cuh"
#include "tc_backward.cuh"
#include "tc_finalize.cuh"
#include "tc_bwd_pipe.cuh"
#include "tc_build_pipe.cuh"
#include "tc_readout_pipe.cuh"
#include "hard_kernels.cuh"

namespace race {

// ------------------------------------------------------------------ NVTX (opt-in)
// With RACE_NVTX=1 in the environment (read once), every entry point and every kernel
// launch of the library is bracketed by an NVTX range named after it, for timeline
// tools.  Off by default: no NVTX call is made.
inline bool nvtx_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("RACE_NVTX");
    return e != nullptr && e[0] == '1';
  }();
  return on;
}

class NvtxRange {
 public:
  explicit NvtxRange(const char* name) : on_(nvtx_enabled()) {
    if (on_) nvtxRangePushA(name);
  }
  ~NvtxRange() {
    if (on_) nvtxRangePop();
  }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;

 private:
  bool on_;
};

// ------------------------------------------------------------------ launch accounting
// Every kernel launch of the library goes through a LaunchScope: it counts launches
// and, while timing is enabled, brackets the launch with CUDA events on its stream.
namespace launches {

std::atomic<int64_t> g_count{0};
std::mutex g_mu;
bool g_timing = false;
struct Timer {
  std::string name;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pending;
  double ms = 0.0;
  int64_t n = 0;
};
std::vector<Timer> g_timers;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

Timer& timer(const char* name) {
  for (auto& t : g_timers)
    if (t.name == name) return t;
  g_timers.push_back(Timer{name, {}, 0.0, 0});
  return g_timers.back();
}

// Resolve pending events into totals (synchronises on them).
void drain() {
  for (auto& t : g_timers) {
    for (auto& pr : t.pending) {
      float ms = 0.f;
      if (cudaEventSynchronize(pr.second) == cudaSuccess &&
          cudaEventElapsedTime(&ms, pr.first, pr.second) == cudaSuccess) {
        t.ms += ms;
        t.n += 1;
      }
      g_pool.push_back(pr.first);
      g_pool.push_back(pr.second);
    }
    t.pending.clear();
  }
}

class Scope {
 public:
  Scope(const char* name, cudaStream_t s) : name_(name), s_(s), range_(name) {
    g_count.fetch_add(1, std::memory_order_relaxed);
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_timing) {
      start_ = take_event();
      stop_ = take_event();
      if (start_ && stop_) cudaEventRecord(start_, s_);
    }
  }
  ~Scope() {
    if (!start_ || !stop_) return;
    std::lock_guard<std::mutex> lk(g_mu);
    cudaEventRecord(stop_, s_);
    timer(name_).pending.emplace_back(start_, stop_);
  }

 private:
  const char* name_;
  cudaStream_t s_;
  NvtxRange range_;
  cudaEvent_t start_ = nullptr, stop_ = nullptr;
};

}  // namespace launches

#define RACE_LAUNCH(name, stream) launches::Scope race_scope_(name, stream)

namespace {

constexpr int kPlanSMs = 148;        // planning constant: SM count of a B200
constexpr size_t kAlign = 256;

inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

race_status_t check_args(const race_args_t* a) {
  if (!a) return RACE_ERR_INVALID_ARG;
  if (a->N < 1 || a->H < 1 || a->L < 1 || a->d < 1) return RACE_ERR_INVALID_ARG;
  if (a->P < 1 || a->P > 8) return RACE_ERR_INVALID_ARG;
  if ((int64_t)a->L * (1 << a->P) > 16384) return RACE_ERR_INVALID_ARG;
  if (!std::isfinite(a->tau) || !(a->tau > 0.f)) return RACE_ERR_INVALID_ARG;
  if (a->causal != 0 && a->causal != 1) return RACE_ERR_INVALID_ARG;
  if ((a->dtype != RACE_BF16 && a->dtype != RACE_FP32) ||
      (a->out_dtype != RACE_BF16 && a->out_dtype != RACE_FP32))
    return RACE_ERR_INVALID_ARG;
  if (a->impl != RACE_IMPL_AUTO && a->impl != RACE_IMPL_SIMT && a->impl != RACE_IMPL_TENSOR)
    return RACE_ERR_INVALID_ARG;
  if (a->grad_dtype != RACE_BF16 && a->grad_dtype != RACE_FP32) return RACE_ERR_INVALID_ARG;
  if (a->w_per_head != 0 && a->w_per_head != 1) return RACE_ERR_INVALID_ARG;
  if (a->chunk < 0 || a->chunk % 32 != 0) return RACE_ERR_INVALID_ARG;
  if ((double)a->N * a->H * a->d > 4.0e18) return RACE_ERR_INVALID_ARG;
  if (a->d != kD) return RACE_ERR_UNSUPPORTED;
  return RACE_OK;
}

Dims dims_of(const race_args_t* a) {
  Dims dm;
  dm.N = a->N;
  dm.H = a->H;
  dm.L = a->L;
  dm.P = a->P;
  dm.R = 1 << a->P;
  dm.tau = a->tau;
  dm.causal = a->causal;
  dm.w_hs = a->w_per_head ? (int64_t)a->L * kD * a->P : 0;
  return dm;
}

// Carried state of race_forward_stream: the public state [H][L*R][65] the sweep starts
// from (in, null = zeros) and the state after the call's tokens (out, may be null).
struct Carry {
  const float* in = nullptr;
  float* out = nullptr;
  bool on = false;
};

// ----------------------------------------------------------------------------- SIMT
struct SimtPlan {
  Dims dm;
  int G;
  int64_t seg_len;
  size_t off_seg, off_init, off_num, off_gpp, off_dxq, off_dxk, off_dv, off_dwq, off_dwk;
  size_t bytes;
};

SimtPlan simt_plan(const race_args_t* a, bool backward) {
  SimtPlan p;
  p.dm = dims_of(a);
  const int64_t tiles = (a->N + simt::TT - 1) / simt::TT;
  int64_t G = (2 * kPlanSMs + (int64_t)a->H * a->L - 1) / ((int64_t)a->H * a->L);
  G = std::max<int64_t>(1, std::min<int64_t>(G, tiles));
  int64_t seg_tiles = (tiles + G - 1) / G;
  p.seg_len = seg_tiles * simt::TT;
  p.G = (int)((a->N + p.seg_len - 1) / p.seg_len);
  const size_t HN = (size_t)a->H * a->N;
  const size_t st = (size_t)a->H * a->L * p.G * p.dm.R * kDV * sizeof(float);
  size_t o = 0;
  p.off_seg = o;  o = align_up(o + st);
  p.off_init = o; o = align_up(o + st);
  p.off_num = o;  o = align_up(o + HN * kNumStride * sizeof(float));
  p.off_gpp = p.off_dxq = p.off_dxk = p.off_dv = p.off_dwq = p.off_dwk = o;
  if (backward) {
    const size_t dwp = (size_t)a->H * a->L * p.G * kD * a->P * sizeof(float);
    p.off_gpp = o; o = align_up(o + HN * kNumStride * sizeof(float));
    p.off_dxq = o; o = align_up(o + HN * kD * sizeof(float));
    p.off_dxk = o; o = align_up(o + HN * kD * sizeof(float));
    p.off_dv = o;  o = align_up(o + HN * kD * sizeof(float));
    p.off_dwq = o; o = align_up(o + dwp);
    p.off_dwk = o; o = align_up(o + dwp);
  }
  p.bytes = o;
  return p;
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)bytes);
}

#define RACE_CU(x)                              \
  do {                                          \
    cudaError_t e_ = (x);                       \
    if (e_ != cudaSuccess) return RACE_ERR_CUDA; \
  } while (0)

// Segment sums and their scan for one side of the sketch (k with [v|1], or q with g'').
template <typename T, int MODE>
race_status_t simt_states(const SimtPlan& p, const T* x, const T* v, const float* gpp,
                          const float* W, char* ws, int scan_mode, cudaStream_t s,
                          const Carry* cy = nullptr) {
  const Dims& dm = p.dm;
  simt::Layout ly(dm.R, dm.P);
  float* seg = reinterpret_cast<float*>(ws + p.off_seg);
  float* init = reinterpret_cast<float*>(ws + p.off_init);
  RACE_CU(set_smem(simt::k_build<T, MODE>, ly.bytes()));
  {
    RACE_LAUNCH("simt_sketch_build", s);
    simt::k_build<T, MODE><<<dim3(p.G, dm.L, dm.H), simt::NT, ly.bytes(), s>>>(
        x, v, gpp, W, seg, dm, p.G, p.seg_len);
  }
  RACE_CU(cudaGetLastError());
  const int RD = dm.R * kDV;
  {
    RACE_LAUNCH("simt_chunk_scan", s);
    if (cy && cy->on)
      simt::k_scan_carry<<<dim3((RD + 255) / 256, dm.H * dm.L), 256, 0, s>>>(
          seg, init, cy->in, cy->out, dm.R, kDV, dm.L, (int64_t)dm.L * dm.R, p.G, scan_mode);
    else
      simt::k_scan<<<dim3((RD + 255) / 256, dm.H * dm.L), 256, 0, s>>>(seg, init, RD, p.G,
                                                                         scan_mode);
  }
  RACE_CU(cudaGetLastError());
  return RACE_OK;
}

template <typename T>
race_status_t simt_forward_num(const SimtPlan& p, const T* q, const T* k, const T* v,
                               const float* W, char* ws, cudaStream_t s,
                               const Carry* cy = nullptr) {
  const Dims& dm = p.dm;
  int have_init = 0;
  if (!dm.causal || p.G > 1 || (cy && cy->on)) {
    race_status_t st =
        simt_states<T, 0>(p, k, v, nullptr, W, ws, dm.causal ? 0 : 2, s, cy);
    if (st != RACE_OK) return st;
    have_init = 1;
  }
  float* num = reinterpret_cast<float*>(ws + p.off_num);
  RACE_CU(cudaMemsetAsync(num, 0, (size_t)dm.H * dm.N * kNumStride * sizeof(float), s));
  simt::Layout ly(dm.R, dm.P);
  RACE_CU(set_smem(simt::k_fwd_sweep<T>, ly.bytes()));
  {
    RACE_LAUNCH("simt_readout_sweep", s);
    simt::k_fwd_sweep<T><<<dim3(p.G, dm.L, dm.H), simt::NT, ly.bytes(), s>>>(
        q, k, v, W, reinterpret_cast<float*>(ws + p.off_init), num, dm, p.G, p.seg_len,
        have_init);
  }
  RACE_CU(cudaGetLastError());
  return RACE_OK;
}

// o = num / den: the vector kernel when the output rows are 16-byte aligned (the
// workspace always is), else one thread per output.
template <typename TO>
void launch_normalize(const float* num, TO* out, float* den, int64_t rows, float inv_L,
                      cudaStream_t s) {
  if ((reinterpret_cast<uintptr_t>(out) & 15) == 0) {
    const int64_t n8 = rows * (kD / 8);
    const int64_t blocks = std::min<int64_t>((n8 + 255) / 256, (int64_t)kPlanSMs * 16);
    simt::k_normalize8<TO><<<(unsigned)std::max<int64_t>(blocks, 1), 256, 0, s>>>(
        num, out, den, rows, inv_L);
  } else {
    simt::k_normalize<TO><<<(unsigned)((rows + 3) / 4), 256, 0, s>>>(num, out, den, rows,
                                                                      inv_L);
  }
}

template <typename T, typename TO>
race_status_t simt_forward(const race_args_t* a, const T* q, const T* k, const T* v,
                           const float* W, TO* out, char* ws, cudaStream_t s,
                           const Carry* cy = nullptr) {
  SimtPlan p = simt_plan(a, false);
  race_status_t st = simt_forward_num<T>(p, q, k, v, W, ws, s, cy);
  if (st != RACE_OK) return st;
  const int64_t rows = (int64_t)a->H * a->N;
  {
    RACE_LAUNCH("simt_normalize", s);
    launch_normalize(reinterpret_cast<float*>(ws + p.off_num), out, a->den, rows, 1.f / a->L, s);
  }
  RACE_CU(cudaGetLastError());
  return RACE_OK;
}

template <typename T, typename TO, typename TG>
race_status_t simt_backward(const race_args_t* a, const T* q, const T* k, const T* v,
                            const float* W, const TO* out, const T* dout, TG* dq, TG* dk,
                            TG* dv, float* dW, char* ws, cudaStream_t s) {
  SimtPlan p = simt_plan(a, true);
  const Dims& dm = p.dm;
  const int64_t rows = (int64_t)a->H * a->N;
  simt::Layout ly(dm.R, dm.P);
  // k-side states (prefix or total), shared by the den recompute and the q sweep
  int have_k = 0;
  if (!dm.causal || p.G > 1) {
    race_status_t st = simt_states<T, 0>(p, k, v, nullptr, W, ws, dm.causal ? 0 : 2, s);
    if (st != RACE_OK) return st;
    have_k = 1;
  }
  float* num = reinterpret_cast<float*>(ws + p.off_num);
  if (!a->den) {
    RACE_CU(cudaMemsetAsync(num, 0, (size_t)rows * kNumStride * sizeof(float), s));
    RACE_CU(set_smem(simt::k_fwd_sweep<T>, ly.bytes()));
    {
      RACE_LAUNCH("simt_readout_sweep", s);
      simt::k_fwd_sweep<T><<<dim3(p.G, dm.L, dm.H), simt::NT, ly.bytes(), s>>>(
          q, k, v, W, reinterpret_cast<float*>(ws + p.off_init), num, dm, p.G, p.seg_len,
          have_k);
    }
    RACE_CU(cudaGetLastError());
  }
  float* gpp = reinterpret_cast<float*>(ws + p.off_gpp);
  {
    RACE_LAUNCH("simt_bwd_prep", s);
    simt::k_gpp<T, TO><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(dout, out, num, a->den,
                                                                   gpp, rows, (float)a->L);
  }
  RACE_CU(cudaGetLastError());
  float* dxq = reinterpret_cast<float*>(ws + p.off_dxq);
  float* dxk = reinterpret_cast<float*>(ws + p.off_dxk);
  float* dva = reinterpret_cast<float*>(ws + p.off_dv);
  RACE_CU(cudaMemsetAsync(dxq, 0, (size_t)rows * kD * sizeof(float), s));
  RACE_CU(cudaMemsetAsync(dxk, 0, (size_t)rows * kD * sizeof(float), s));
  RACE_CU(cudaMemsetAsync(dva, 0, (size_t)rows * kD * sizeof(float), s));
  float* dwq = reinterpret_cast<float*>(ws + p.off_dwq);
  float* dwk = reinterpret_cast<float*>(ws + p.off_dwk);
  RACE_CU(set_smem(simt::k_bwd_q<T>, ly.bytes()));
  {
    RACE_LAUNCH("simt_bwd_q", s);
    simt::k_bwd_q<T><<<dim3(p.G, dm.L, dm.H), simt::NT, ly.bytes(), s>>>(
        q, k, v, W, reinterpret_cast<float*>(ws + p.off_init), gpp, dxq, dwq, dm, p.G,
        p.seg_len, have_k);
  }
  RACE_CU(cudaGetLastError());
  int have_q = 0;
  if (!dm.causal || p.G > 1) {
    race_status_t st = simt_states<T, 1>(p, q, v, gpp, W, ws, dm.causal ? 1 : 2, s);
    if (st != RACE_OK) return st;
    have_q = 1;
  }
  RACE_CU(set_smem(simt::k_bwd_kv<T>, ly.bytes()));
  {
    RACE_LAUNCH("simt_bwd_kv", s);
    simt::k_bwd_kv<T><<<dim3(p.G, dm.L, dm.H), simt::NT, ly.bytes(), s>>>(
        q, k, v, W, reinterpret_cast<float*>(ws + p.off_init), gpp, dxk, dva, dwk, dm, p.G,
        p.seg_len, have_q);
  }
  RACE_CU(cudaGetLastError());
  {
    RACE_LAUNCH("simt_bwd_finalize_dx", s);
    simt::k_finalize_dx<T, TG><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(q, dxq, dq, rows);
  }
  {
    RACE_LAUNCH("simt_bwd_finalize_dx", s);
    simt::k_finalize_dx<T, TG><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(k, dxk, dk, rows);
  }
  {
    RACE_LAUNCH("simt_bwd_convert_dv", s);
    simt::k_convert<TG><<<1184, 256, 0, s>>>(dva, dv, rows * kD);
  }
  const int nW = (a->w_per_head ? a->H : 1) * a->L * kD * a->P;
  {
    RACE_LAUNCH("simt_dW_reduce", s);
    simt::k_dw_reduce<<<(nW + 255) / 256, 256, 0, s>>>(dwq, dwk, dW, a->H, a->L, p.G, a->P,
                                                       a->w_per_head);
  }
  RACE_CU(cudaGetLastError());
  return RACE_OK;
}

bool use_tensor_path(const race_args_t* a) {
  if (a->impl == RACE_IMPL_SIMT) return false;
  if (a->dtype != RACE_BF16) return false;
  return tc::supported(a);
}

bool tc_backward_supported(const race_args_t* a);
struct BwPlan;
size_t bw_plan_bytes(const race_args_t* a);

bool use_tensor_backward(const race_args_t* a) {
  if (a->impl == RACE_IMPL_SIMT) return false;
  if (a->dtype != RACE_BF16) return false;
  return tc_backward_supported(a);
}

size_t workspace_bytes(const race_args_t* a, bool backward) {
  if (!backward && use_tensor_path(a)) return tc::forward_workspace(a);
  if (backward && use_tensor_backward(a)) return bw_plan_bytes(a);
  return simt_plan(a, backward).bytes;
}

// ----------------------------------------------------------------------------- tensor
template <int P>
race_status_t tc_launch(int mode, const tc::Params& prm, const CUtensorMap& tq,
                        const CUtensorMap& tk, const CUtensorMap& tv, const float* W,
                        const float* init, float* seg, float* num, const float* inv_norms,
                        int64_t inv_stride, const float* kscale, cudaStream_t s) {
  dim3 grid(prm.G, prm.n_rg, prm.H);
  const size_t smem = tc::Smem::alloc;
#define RACE_TC(MODE, NAME)                                                        \
  do {                                                                             \
    RACE_CU(set_smem(tc::k_sketch<P, MODE>, smem));                                \
    RACE_LAUNCH(NAME, s);                                                          \
    tc::k_sketch<P, MODE><<<grid, tc::kThreads, smem, s>>>(tq, tk, tv, W, init, seg, \
                                                            num, kscale, prm);     \
  } while (0)
  if (mode == tc::kSweep && P == 8 && prm.rows == 256 && inv_norms) {
    CUtensorMap tnum;
    if (!tc::encode_num_tmap(&tnum, num, prm.N, prm.H)) return RACE_ERR_CUDA;
    // A per-key factor means the backward's dv pass, which reads only the 64 value
    // columns of num: the sweep then runs its value-side MMAs at N = 64 (no mass column).
    auto* kern = kscale ? tc::k_sweep_pipe<64> : tc::k_sweep_pipe<80>;
    RACE_CU(set_smem(kern, tc::SPSmem::alloc));
    RACE_LAUNCH("tc_causal_sweep", s);
    kern<<<grid, tc::kSPThreads, tc::SPSmem::alloc, s>>>(tq, tk, tv, W, init, inv_norms,
                                                        inv_stride, tnum, num, kscale, prm);
  } else if (mode == tc::kSweep && prm.rows == 256) {
    constexpr int TABLES = 256 >> P;
    RACE_CU(set_smem(tc::k_sweep<P, TABLES>, tc::SwSmem::alloc));
    RACE_LAUNCH("tc_causal_sweep", s);
    tc::k_sweep<P, TABLES><<<grid, tc::kSwThreads, tc::SwSmem::alloc, s>>>(tq, tk, tv, W, init,
                                                                          num, kscale, prm);
  } else if (mode == tc::kSweep) RACE_TC(tc::kSweep, "tc_causal_sweep_rows128");
  else if (mode == tc::kBuild && P < 8 && prm.rows == 256 && !prm.have_init) {
    if constexpr (P < 8) {
      RACE_CU(set_smem(tc::k_build_pipe<P>, tc::BldSmem::alloc));
      RACE_LAUNCH("tc_sketch_build", s);
      tc::k_build_pipe<P><<<grid, tc::kBPipeThreads, tc::BldSmem::alloc, s>>>(tk, tv, W, seg,
                                                                             kscale, prm);
    }
  } else if (mode == tc::kBuild) RACE_TC(tc::kBuild, "tc_sketch_build");
  else if (P < 8 && prm.rows == 256 && prm.have_init) {
    if constexpr (P < 8) {
      RACE_CU(set_smem(tc::k_readout_pipe<P>, tc::RdSmem::alloc));
      RACE_LAUNCH("tc_readout", s);
      tc::k_readout_pipe<P><<<grid, tc::kRPipeThreads, tc::RdSmem::alloc, s>>>(tq, W, init,
                                                                              num, prm);
    }
  } else RACE_TC(tc::kReadout, "tc_readout");
#undef RACE_TC
  RACE_CU(cudaGetLastError());
  return RACE_OK;
}

race_status_t tc_dispatch(int P, int mode, const tc::Params& prm, const CUtensorMap& tq,
                          const CUtensorMap& tk, const CUtensorMap& tv, const float* W,
                          const float* init, float* seg, float* num, const float* kscale,
                          cudaStream_t s, const float* inv_norms = nullptr,
                          int64_t inv_stride = 0) {
  switch (P) {
    case 6: return tc_launch<6>(mode, prm, tq, tk, tv, W, init, seg, num, inv_norms, inv_stride, kscale, s);
    case 7: return tc_launch<7>(mode, prm, tq, tk, tv, W, init, seg, num, inv_norms, inv_stride, kscale, s);
    case 8: return tc_launch<8>(mode, prm, tq, tk, tv, W, init, seg, num, inv_norms, inv_stride, kscale, s);
  }
  return RACE_ERR_UNSUPPORTED;
}

// Forward accumulators num[h][n][0..64] (unnormalised, den' in column 64) in the
// forward plan's scratch.  kscale (nullable, [H][N] float32) multiplies every p(k_n):
// the backward's dv pass runs this with the keys' 1/den'.
race_status_t tc_forward_num(const race_args_t* a, const void* q, const void* k, const void* v,
                             const float* W, char* ws, float** num_out, cudaStream_t s,
                             const float* kscale = nullptr, const Carry* cy = nullptr) {
  tc::Plan pl = tc::make_plan(a);
  CUtensorMap tq, tk, tv;
  if (!tc::encode_tmap(&tq, q, a->N, a->H) || !tc::encode_tmap(&tk, k, a->N, a->H) ||
      !tc::encode_tmap(&tv, v, a->N, a->H))
    return RACE_ERR_CUDA;
  float* num = reinterpret_cast<float*>(ws + pl.off_num);
  float* seg = reinterpret_cast<float*>(ws + pl.off_seg);
  float* init = reinterpret_cast<float*>(ws + pl.off_init);
  const int64_t rows = (int64_t)a->H * a->N;
  RACE_CU(cudaMemsetAsync(num, 0, (size_t)rows * kNumStride * sizeof(float), s));
  tc::Params prm = pl.prm;
  race_status_t st;
  const bool carry = cy && cy->on;
  if (!a->causal || prm.G > 1 || carry) {
    st = tc_dispatch(pl.P, tc::kBuild, prm, tq, tk, tv, W, init, seg, num, kscale, s);
    if (st != RACE_OK) return st;
    const int RD = prm.rows * tc::kNV;
    {
      RACE_LAUNCH("tc_chunk_scan", s);
      if (carry)
        simt::k_scan_carry<<<dim3((RD + 255) / 256, prm.H * prm.n_rg), 256, 0, s>>>(
            seg, init, cy->in, cy->out, prm.rows, tc::kNV, prm.n_rg, (int64_t)prm.L * prm.R,
            prm.G, a->causal ? 0 : 2);
      else
        simt::k_scan<<<dim3((RD + 255) / 256, prm.H * prm.n_rg), 256, 0, s>>>(
            seg, init, RD, prm.G, a->causal ? 0 : 2);
    }
    RACE_CU(cudaGetLastError());
    prm.have_init = 1;
  }
  float* inv_norms = nullptr;
  if (a->causal && pl.P == 8 && prm.rows == 256) {
    inv_norms = reinterpret_cast<float*>(ws + pl.off_inv);
    RACE_LAUNCH("tc_inv_norms", s);
    tc::k_inv_norms<<<dim3((unsigned)((a->N + 127) / 128), 2 * a->H), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), inv_norms,
        a->N, a->H, pl.inv_stride);
  }
  RACE_CU(cudaGetLastError());
  st = tc_dispatch(pl.P, a->causal ? tc::kSweep : tc::kReadout, prm, tq, tk, tv, W, init,
                   seg, num, kscale, s, inv_norms, pl.inv_stride);
  if (st != RACE_OK) return st;
  *num_out = num;
  return RACE_OK;
}

template <typename TO>
race_status_t tc_forward(const race_args_t* a, const void* q, const void* k, const void* v,
                         const float* W, TO* out, char* ws, cudaStream_t s,
                         const Carry* cy = nullptr) {
  float* num = nullptr;
  race_status_t st = tc_forward_num(a, q, k, v, W, ws, &num, s, nullptr, cy);
  if (st != RACE_OK) return st;
  const int64_t rows = (int64_t)a->H * a->N;
  {
    RACE_LAUNCH("tc_normalize", s);
    launch_normalize(num, out, a->den, rows, 1.f / a->L, s);
  }
  RACE_CU(cudaGetLastError());
  return RACE_OK;
}

// ----------------------------------------------------------------------------- tensor backward
// Row groups of 256 sketch rows (L*R a multiple of 256) and L*P <= 256.
bool tc_backward_supported(const race_args_t* a) {
  if (!tc::supported(a)) return false;
  const int64_t LR = (int64_t)a->L << a->P;
  return LR % 256 == 0 && (int64_t)a->L * a->P <= tc::kMaxLP;
}

// The causal sweeps at R = 256 run as the pipelined kernel k_bwd_pipe (two CTAs per table).
bool bw_pipelined(const race_args_t* a) { return a->P == 8 && a->causal; }

struct BwPlan {
  tc::Params prm;
  int fin_blocks;
  bool pipe;                 // k_bwd_pipe for the q and k sweeps
  int64_t inv_stride;        // row stride of the 1/|x| scratch (whole chunks)
  size_t off_fwd, off_rinv, off_gdot, off_rq, off_rk, off_rg, off_rr, off_duq, off_duk,
      off_seg, off_init, off_part, off_inv, off_z, off_gext, bytes;
};

BwPlan make_bw_plan(const race_args_t* a) {
  BwPlan b;
  tc::Params& p = b.prm;
  p.N = a->N;
  p.H = a->H;
  p.L = a->L;
  p.R = 1 << a->P;
  p.rows = 256;
  p.tables = 256 / p.R;
  p.np = ((p.tables * a->P + 15) / 16) * 16;
  p.n_rg = (a->L * p.R) / 256;
  b.pipe = bw_pipelined(a);
  // CTAs per (head, segment): one per row group, two per table for the pipelined sweep
  const int64_t units = (int64_t)a->H * p.n_rg * (b.pipe ? 2 : 1);
  const int64_t tiles = (a->N + tc::kC - 1) / tc::kC;
  int64_t G = a->causal ? std::max<int64_t>(1, kPlanSMs / units)
                        : std::max<int64_t>(1, (kPlanSMs + units - 1) / units);
  G = std::min<int64_t>(G, tiles);
  p.seg_len = ((tiles + G - 1) / G) * tc::kC;
  p.G = (int)((a->N + p.seg_len - 1) / p.seg_len);
  p.two_over_tau = 2.0f / a->tau;
  p.have_init = 0;
  const int64_t rows = (int64_t)a->H * a->N;
  const int LP = a->L * a->P;
  p.lps = (LP + 7) / 8 * 8;   // 16-byte rows of bf16 per-plane gradients
  p.w_hs = a->w_per_head ? (int64_t)LP * kD : 0;
  // finalize blocks per head: at most one CTA per SM over all heads (tensor-core finalize,
  // 128-token tiles, one resident CTA per SM) or four (CUDA-core finalize, 64-token tiles),
  // rounded down so that the grid is a single wave
  {
    const int tile = LP <= tc::kFzMaxLP ? 128 : tc::kFinTok;
    const int64_t per_sm = LP <= tc::kFzMaxLP ? 1 : 4;
    const int64_t want = std::max<int64_t>(1, per_sm * kPlanSMs / a->H);
    b.fin_blocks = (int)std::max<int64_t>(1, std::min<int64_t>(want, (a->N + tile - 1) / tile));
  }
  const size_t st = (size_t)a->H * p.n_rg * p.G * 256 * tc::kNV * sizeof(float);
  const size_t xb = (size_t)rows * kD * sizeof(__nv_bfloat16);
  size_t o = 0;
  b.off_fwd = o;  o = align_up(o + tc::forward_workspace(a));
  b.off_rinv = o; o = align_up(o + (size_t)rows * sizeof(float));
  b.off_gdot = o; o = align_up(o + (size_t)rows * sizeof(float));
  b.off_rq = b.off_rk = b.off_rg = b.off_rr = o;
  if (a->causal) {
    b.off_rq = o; o = align_up(o + xb);
    b.off_rk = o; o = align_up(o + xb);
    b.off_rg = o; o = align_up(o + xb);
    b.off_rr = o; o = align_up(o + (size_t)rows * sizeof(float));
  }
  // per-plane gradients du' of each side: bf16 hi array then bf16 lo array, [rows][lps]
  b.off_duq = o;  o = align_up(o + 2 * (size_t)rows * p.lps * sizeof(__nv_bfloat16));
  b.off_duk = o;  o = align_up(o + 2 * (size_t)rows * p.lps * sizeof(__nv_bfloat16));
  b.off_seg = o;  o = align_up(o + st);
  b.off_init = o; o = align_up(o + st);
  b.off_part = o; o = align_up(o + 2 * (size_t)a->H * b.fin_blocks * LP * kD * sizeof(float));
  // 1/|x| of q and k rows, [2][H][inv_stride], and their scaled projections,
  // [2][H][L][inv_stride][8] (pipelined sweep only)
  b.inv_stride = tiles * tc::kC;
  b.off_inv = o;
  if (b.pipe) o = align_up(o + 2 * (size_t)a->H * b.inv_stride * sizeof(float));
  b.off_z = o;
  if (b.pipe) o = align_up(o + 2 * (size_t)a->H * a->L * b.inv_stride * 8 * sizeof(float));
  // extra feature columns of g', [H][N][16] bf16 (pipelined sweep only)
  b.off_gext = o;
  if (b.pipe) o = align_up(o + (size_t)rows * 16 * sizeof(__nv_bfloat16));
  b.bytes = o;
  return b;
}

size_t bw_plan_bytes(const race_args_t* a) { return make_bw_plan(a).bytes; }

template <int P>
race_status_t bw_launch(int mode, bool rev, const tc::Params& prm, const CUtensorMap& xa,
                        const CUtensorMap& xb, const CUtensorMap& fa, const CUtensorMap& fb,
                        const float* ea, const float* eb, const float* ra, const float* rb,
                        const float* W, const float* init, float* seg, __nv_bfloat16* du,
                        const char* name, cudaStream_t s) {
  dim3 grid(prm.G, prm.n_rg, prm.H);
  const size_t smem = tc::BwSmem::alloc;
#define RACE_BW(MODE, REV)                                                                 \
  do {                                                                                     \
    RACE_CU(set_smem(tc::k_bwd_phi<P, MODE, REV>, smem));                                  \
    RACE_LAUNCH(name, s);                                                                  \
    tc::k_bwd_phi<P, MODE, REV><<<grid, tc::kBwThreads, smem, s>>>(                        \
        xa, xb, fa, fb, ea, eb, ra, rb, W, init, seg, du, prm);                            \
  } while (0)
  if (mode == tc::kBuild) RACE_BW(tc::kBuild, false);
  else if (mode == tc::kReadout) RACE_BW(tc::kReadout, false);
  else if (rev) RACE_BW(tc::kSweep, true);
  else RACE_BW(tc::kSweep, false);
#undef RACE_BW
  RACE_CU(cudaGetLastError());
  return RACE_OK;
}

race_status_t bw_dispatch(int P, int mode, bool rev, const tc::Params& prm,
                          const CUtensorMap& xa, const CUtensorMap& xb, const CUtensorMap& fa,
                          const CUtensorMap& fb, const float* ea, const float* eb,
                          const float* ra, const float* rb, const float* W, const float* init,
                          float* seg, __nv_bfloat16* du, const char* name, cudaStream_t s) {
  switch (P) {
    case 6: return bw_launch<6>(mode, rev, prm, xa, xb, fa, fb, ea, eb, ra, rb, W, init, seg, du, name, s);
    case 7: return bw_launch<7>(mode, rev, prm, xa, xb, fa, fb, ea, eb, ra, rb, W, init, seg, du, name, s);
    case 8: return bw_launch<8>(mode, rev, prm, xa, xb, fa, fb, ea, eb, ra, rb, W, init, seg, du, name, s);
  }
  return RACE_ERR_UNSUPPORTED;
}

// The pipelined causal sweep at R = 256: grid (G, 2 * tables, H) in clusters of the two
// halves of a table.
race_status_t bw_pipe_launch(bool rev, const tc::Params& prm, const CUtensorMap& fa,
                             const CUtensorMap& fb, const CUtensorMap& ge, const float* rinv,
                             const float* za, const float* zb, const float* inv_a,
                             int64_t zstride, const float* init, __nv_bfloat16* du,
                             const char* name, cudaStream_t s) {
  const dim3 grid(prm.G, 2 * prm.n_rg, prm.H);
  const size_t smem = tc::BPSmem::alloc;
  if (rev) {
    RACE_CU(set_smem(tc::k_bwd_pipe<true>, smem));
    RACE_LAUNCH(name, s);
    tc::k_bwd_pipe<true><<<grid, tc::kBPThreads, smem, s>>>(fa, fb, ge, rinv, za, zb, inv_a,
                                                             zstride, init, du, prm);
  } else {
    RACE_CU(set_smem(tc::k_bwd_pipe<false>, smem));
    RACE_LAUNCH(name, s);
    tc::k_bwd_pipe<false><<<grid, tc::kBPThreads, smem, s>>>(fa, fb, ge, rinv, za, zb, inv_a,
                                                              zstride, init, du, prm);
  }
  RACE_CU(cudaGetLastError());
  return RACE_OK;
}

template <int MT, typename TG>
race_status_t finalize_launch_mt(const __nv_bfloat16* x, const __nv_bfloat16* du,
                                 const float* W, TG* dx, float* part, int64_t N, int H, int L,
                                 int P, int lps, int64_t w_hs, int blocks, size_t fsm,
                                 cudaStream_t s) {
  RACE_CU(set_smem(tc::k_bwd_finalize<__nv_bfloat16, MT, TG>, fsm));
  RACE_LAUNCH("tc_bwd_finalize", s);
  tc::k_bwd_finalize<__nv_bfloat16, MT, TG><<<dim3(blocks, H), 256, fsm, s>>>(
      x, du, W, dx, part, N, L, P, lps, w_hs);
  RACE_CU(cudaGetLastError());
  return RACE_OK;
}

// dx and the dW partials [H][blocks][L*P][64] of one side from its per-plane gradients du'
// (bf16 hi + lo): on tensor cores for L*P <= 128, else on CUDA cores (MT = ceil(L*P/16)).
template <typename TG>
race_status_t finalize_side(const __nv_bfloat16* x, const __nv_bfloat16* du, const float* W,
                            TG* dx, float* part, int64_t N, int H, int L, int P, int lps,
                            int64_t w_hs, int blocks, cudaStream_t s) {
  const int LP = L * P;
  if (LP <= tc::kFzMaxLP) {
    CUtensorMap tduh, tdul, tx;
    if (!tc::encode_rows_bf16(&tduh, du, LP, N, H, lps) ||
        !tc::encode_rows_bf16(&tdul, du + (size_t)H * N * lps, LP, N, H, lps) ||
        !tc::encode_tmap(&tx, x, N, H))
      return RACE_ERR_CUDA;
    RACE_CU(set_smem(tc::k_bwd_finalize_tc<TG>, tc::FzSmem::alloc));
    RACE_LAUNCH("tc_bwd_finalize", s);
    tc::k_bwd_finalize_tc<TG><<<dim3(blocks, H), tc::kFzThreads, tc::FzSmem::alloc, s>>>(
        tduh, tdul, tx, W, dx, part, N, L, P, w_hs);
    RACE_CU(cudaGetLastError());
    return RACE_OK;
  }
  const size_t fsm = tc::finalize_smem(LP);
#define RACE_FIN(M) \
  case M:           \
    return finalize_launch_mt<M, TG>(x, du, W, dx, part, N, H, L, P, lps, w_hs, blocks, fsm, s)
  switch (tc::finalize_mt(LP)) {
    RACE_FIN(1); RACE_FIN(2); RACE_FIN(3); RACE_FIN(4); RACE_FIN(5); RACE_FIN(6); RACE_FIN(7);
    RACE_FIN(8); RACE_FIN(9); RACE_FIN(10); RACE_FIN(11); RACE_FIN(12); RACE_FIN(13);
    RACE_FIN(14); RACE_FIN(15); RACE_FIN(16);
  }
#undef RACE_FIN
  return RACE_ERR_UNSUPPORTED;
}

template <typename TO, typename TG>
race_status_t tc_backward(const race_args_t* a, const __nv_bfloat16* q, const __nv_bfloat16* k,
                          const __nv_bfloat16* v, const float* W, const TO* out,
                          const __nv_bfloat16* dout, TG* dq, TG* dk, TG* dv, float* dW,
                          char* ws, cudaStream_t s) {
  const BwPlan pl = make_bw_plan(a);
  const int64_t rows = (int64_t)a->H * a->N;
  const int LP = a->L * a->P;
  char* fws = ws + pl.off_fwd;
  float* rinv = reinterpret_cast<float*>(ws + pl.off_rinv);
  float* gdot = reinterpret_cast<float*>(ws + pl.off_gdot);
  auto* duq = reinterpret_cast<__nv_bfloat16*>(ws + pl.off_duq);
  auto* duk = reinterpret_cast<__nv_bfloat16*>(ws + pl.off_duk);
  float* seg = reinterpret_cast<float*>(ws + pl.off_seg);
  float* init = reinterpret_cast<float*>(ws + pl.off_init);
  float* partq = reinterpret_cast<float*>(ws + pl.off_part);
  float* partk = partq + (size_t)a->H * pl.fin_blocks * LP * kD;
  race_status_t st;
  // ---- den' (recomputed by a forward when not saved), -(g . o) and 1/den'
  float* num = nullptr;
  if (!a->den) {
    st = tc_forward_num(a, q, k, v, W, fws, &num, s);
    if (st != RACE_OK) return st;
  }
  {
    RACE_LAUNCH("tc_bwd_prep", s);
    const int64_t blocks = std::min<int64_t>((rows + 31) / 32, (int64_t)kPlanSMs * 16);
    tc::k_bwd_prep<__nv_bfloat16, TO><<<(unsigned)blocks, 256, 0, s>>>(
        dout, out, num, a->den, gdot, rinv, rows, (float)a->L);
  }
  RACE_CU(cudaGetLastError());
  // g enters the feature tiles exactly as given (bf16 upstream gradient)
  CUtensorMap xq, xk, fv, fg;
  if (!tc::encode_tmap(&xq, q, a->N, a->H) || !tc::encode_tmap(&xk, k, a->N, a->H) ||
      !tc::encode_feat_tmap(&fv, v, a->N, a->H) || !tc::encode_feat_tmap(&fg, dout, a->N, a->H))
    return RACE_ERR_CUDA;
  const int mode = a->causal ? tc::kSweep : tc::kReadout;
  const int RD = 256 * tc::kNV;
  float* inv_q = reinterpret_cast<float*>(ws + pl.off_inv);
  float* inv_k = inv_q + (size_t)a->H * pl.inv_stride;
  float* z_q = reinterpret_cast<float*>(ws + pl.off_z);
  float* z_k = z_q + (size_t)a->H * a->L * pl.inv_stride * 8;
  auto* gext = reinterpret_cast<__nv_bfloat16*>(ws + pl.off_gext);
  CUtensorMap tge;
  if (pl.pipe) {
    {
      const size_t zsm = tc::zproj_smem(a->L);
      const int per_sm = 512 / tc::zproj_cols(a->L);
      const int64_t tiles = (a->N + tc::kC - 1) / tc::kC;
      const int64_t want = std::max<int64_t>(1, (int64_t)kPlanSMs * per_sm / (2 * a->H));
      const unsigned gx = (unsigned)std::min<int64_t>(tiles, want);
      RACE_CU(set_smem(tc::k_bwd_zproj, zsm));
      RACE_LAUNCH("tc_bwd_zproj", s);
      tc::k_bwd_zproj<<<dim3(gx, a->H, 2), tc::kZpThreads, zsm, s>>>(
          xq, xk, W, pl.prm.w_hs, z_q, inv_q, a->N, a->H, a->L, pl.inv_stride,
          pl.prm.two_over_tau);
    }
    RACE_CU(cudaGetLastError());
    {
      RACE_LAUNCH("tc_bwd_gext", s);
      tc::k_bwd_gext<<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(gdot, gext, rows);
    }
    RACE_CU(cudaGetLastError());
    if (!tc::encode_gext_tmap(&tge, gext, a->N, a->H)) return RACE_ERR_CUDA;
  }
  // ---- q side: dP(q) = r (g' S^T + mask(g' [v|1]^T) p(k)), S over keys j <= i
  tc::Params prm = pl.prm;
  if (!a->causal || prm.G > 1) {
    st = bw_dispatch(a->P, tc::kBuild, false, prm, xk, xk, fv, fv, nullptr, nullptr, nullptr,
                     nullptr, W, init, seg, nullptr, "tc_bwd_build_k", s);
    if (st != RACE_OK) return st;
    {
      RACE_LAUNCH("tc_chunk_scan", s);
      simt::k_scan<<<dim3((RD + 255) / 256, prm.H * prm.n_rg), 256, 0, s>>>(
          seg, init, RD, prm.G, a->causal ? 0 : 2);
    }
    RACE_CU(cudaGetLastError());
    prm.have_init = 1;
  }
  st = pl.pipe ? bw_pipe_launch(false, prm, fg, fv, tge, rinv, z_q, z_k, inv_q,
                                pl.inv_stride, init, duq, "tc_bwd_q", s)
               : bw_dispatch(a->P, mode, false, prm, xq, xk, fg, fv, gdot, nullptr, rinv,
                             nullptr, W, init, seg, duq, "tc_bwd_q", s);
  if (st != RACE_OK) return st;
  // ---- k side: dP(k) = [v|1] T^T + mask([v|1] g'^T) (r p(q)), T over queries i >= j
  prm = pl.prm;
  if (!a->causal || prm.G > 1) {
    st = bw_dispatch(a->P, tc::kBuild, false, prm, xq, xq, fg, fg, nullptr, gdot, nullptr,
                     rinv, W, init, seg, nullptr, "tc_bwd_build_q", s);
    if (st != RACE_OK) return st;
    {
      RACE_LAUNCH("tc_chunk_scan", s);
      simt::k_scan<<<dim3((RD + 255) / 256, prm.H * prm.n_rg), 256, 0, s>>>(
          seg, init, RD, prm.G, a->causal ? 1 : 2);
    }
    RACE_CU(cudaGetLastError());
    prm.have_init = 1;
  }
  st = pl.pipe ? bw_pipe_launch(true, prm, fv, fg, tge, rinv, z_k, z_q, inv_k,
                                pl.inv_stride, init, duk, "tc_bwd_k", s)
               : bw_dispatch(a->P, mode, a->causal != 0, prm, xk, xq, fv, fg, nullptr, gdot,
                             nullptr, rinv, W, init, seg, duk, "tc_bwd_k", s);
  if (st != RACE_OK) return st;
  // ---- dv_j = sum_{i >= j} w_ij r_i g_i: the forward sweep with queries k, keys q (each
  //      p(q_i) scaled by r_i) and values g (sequence reversed for the causal case)
  race_args_t av = *a;
  av.den = nullptr;
  float* vnum = nullptr;
  if (a->causal) {
    auto* rq = reinterpret_cast<__nv_bfloat16*>(ws + pl.off_rq);
    auto* rk = reinterpret_cast<__nv_bfloat16*>(ws + pl.off_rk);
    auto* rg = reinterpret_cast<__nv_bfloat16*>(ws + pl.off_rg);
    float* rr = reinterpret_cast<float*>(ws + pl.off_rr);
    const unsigned blocks = (unsigned)((rows * 8 + 255) / 256);
    {
      RACE_LAUNCH("tc_bwd_reverse", s);
      tc::k_reverse_rows<<<blocks, 256, 0, s>>>(q, rq, a->N, a->H);
      tc::k_reverse_rows<<<blocks, 256, 0, s>>>(k, rk, a->N, a->H);
      tc::k_reverse_rows<<<blocks, 256, 0, s>>>(dout, rg, a->N, a->H);
      tc::k_reverse_vec<<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(rinv, rr, a->N, a->H);
    }
    RACE_CU(cudaGetLastError());
    st = tc_forward_num(&av, rk, rq, rg, W, fws, &vnum, s, rr);
  } else {
    st = tc_forward_num(&av, k, q, dout, W, fws, &vnum, s, rinv);
  }
  if (st != RACE_OK) return st;
  {
    RACE_LAUNCH("tc_bwd_dv_out", s);
    tc::k_dv_out<TG><<<dim3((unsigned)((a->N + 15) / 16), a->H), 256, 0, s>>>(
        vnum, dv, a->N, a->H, a->causal);
  }
  RACE_CU(cudaGetLastError());
  // ---- dq, dk through the projections and the normalisation; dW
  st = finalize_side(q, duq, W, dq, partq, a->N, a->H, a->L, a->P, pl.prm.lps, pl.prm.w_hs,
                     pl.fin_blocks, s);
  if (st != RACE_OK) return st;
  st = finalize_side(k, duk, W, dk, partk, a->N, a->H, a->L, a->P, pl.prm.lps, pl.prm.w_hs,
                     pl.fin_blocks, s);
  if (st != RACE_OK) return st;
  const int nW = (a->w_per_head ? a->H : 1) * a->L * kD * a->P;
  {
    RACE_LAUNCH("tc_bwd_dW_reduce", s);
    tc::k_bwd_dw_reduce<<<(nW + 255) / 256, 256, 0, s>>>(partq, partk, a->H, pl.fin_blocks,
                                                         a->w_per_head, dW, a->L, a->P);
  }
  RACE_CU(cudaGetLastError());
  return RACE_OK;
}

// ----------------------------------------------------------------------------- hard hash
// Classic RACE with hard P-bit hashes (hard_kernels.cuh): scratch layout and launches.
struct HardPlan {
  int G;
  int64_t seg_len;
  size_t off_qid, off_kid, off_cseg, off_cinit, off_vseg, off_vinit, off_num, off_cnt, bytes;
};

HardPlan hard_plan(const race_args_t* a) {
  HardPlan p;
  const int R = 1 << a->P;
  const int64_t chunks = (a->N + hard::kHC - 1) / hard::kHC;
  const int64_t units = (int64_t)a->H * a->L;
  int64_t G = std::max<int64_t>(1, (2 * kPlanSMs + units - 1) / units);
  G = std::min<int64_t>(G, chunks);
  p.seg_len = ((chunks + G - 1) / G) * hard::kHC;
  p.G = (int)((a->N + p.seg_len - 1) / p.seg_len);
  const size_t rows = (size_t)a->H * a->N;
  const size_t cells = (size_t)a->H * a->L * p.G * R;
  size_t o = 0;
  p.off_qid = o;   o = align_up(o + rows * a->L);
  p.off_kid = o;   o = align_up(o + rows * a->L);
  p.off_cseg = o;  o = align_up(o + cells * sizeof(int));
  p.off_cinit = o; o = align_up(o + cells * sizeof(int));
  p.off_vseg = o;  o = align_up(o + cells * kD * sizeof(float));
  p.off_vinit = o; o = align_up(o + cells * kD * sizeof(float));
  p.off_num = o;   o = align_up(o + rows * kD * sizeof(float));
  p.off_cnt = o;   o = align_up(o + rows * sizeof(int));
  p.bytes = o;
  return p;
}

template <typename T>
race_status_t hard_ids(const race_args_t* a, const T* x, const float* W, uint8_t* ids,
                       cudaStream_t s) {
  const int64_t w_hs = a->w_per_head ? (int64_t)a->L * kD * a->P : 0;
  RACE_LAUNCH("hard_ids", s);
  hard::k_hard_ids<T><<<dim3((unsigned)((a->N + 31) / 32), a->H), hard::kHT, 0, s>>>(
      x, W, ids, a->N, a->L, a->P, w_hs);
  RACE_CU(cudaGetLastError());
  return RACE_OK;
}

template <typename T, typename TO>
race_status_t hard_forward(const race_args_t* a, const T* q, const T* k, const T* v,
                           const float* W, TO* out, int* counts, char* ws, cudaStream_t s) {
  const HardPlan p = hard_plan(a);
  const int R = 1 << a->P;
  auto* qid = reinterpret_cast<uint8_t*>(ws + p.off_qid);
  auto* kid = reinterpret_cast<uint8_t*>(ws + p.off_kid);
  int* cseg = reinterpret_cast<int*>(ws + p.off_cseg);
  int* cinit = reinterpret_cast<int*>(ws + p.off_cinit);
  float* vseg = reinterpret_cast<float*>(ws + p.off_vseg);
  float* vinit = reinterpret_cast<float*>(ws + p.off_vinit);
  float* num = reinterpret_cast<float*>(ws + p.off_num);
  int* cnt = counts ? counts : reinterpret_cast<int*>(ws + p.off_cnt);
  const size_t rows = (size_t)a->H * a->N;
  race_status_t st = hard_ids<T>(a, q, W, qid, s);
  if (st != RACE_OK) return st;
  st = hard_ids<T>(a, k, W, kid, s);
  if (st != RACE_OK) return st;
  RACE_CU(cudaMemsetAsync(num, 0, rows * kD * sizeof(float), s));
  RACE_CU(cudaMemsetAsync(cnt, 0, rows * sizeof(int), s));
  const dim3 grid(p.G, a->L, a->H);
  int have_init = 0;
  if (!a->causal || p.G > 1) {
    RACE_CU(set_smem(hard::k_hard_seg<T>, hard::seg_smem(R)));
    {
      RACE_LAUNCH("hard_segments", s);
      hard::k_hard_seg<T><<<grid, hard::kHT, hard::seg_smem(R), s>>>(kid, v, cseg, vseg, a->N,
                                                                    a->L, R, p.G, p.seg_len);
    }
    RACE_CU(cudaGetLastError());
    {
      RACE_LAUNCH("hard_scan", s);
      hard::k_hard_scan<<<dim3((R * kDV + 255) / 256, a->H * a->L), 256, 0, s>>>(
          cseg, vseg, cinit, vinit, R, p.G, a->causal ? 0 : 2);
    }
    RACE_CU(cudaGetLastError());
    have_init = 1;
  }
  RACE_CU(set_smem(hard::k_hard_sweep<T>, hard::sweep_smem(R)));
  {
    RACE_LAUNCH("hard_sweep", s);
    hard::k_hard_sweep<T><<<grid, hard::kHT, hard::sweep_smem(R), s>>>(
        qid, kid, v, cinit, vinit, num, cnt, a->N, a->L, R, p.G, p.seg_len, a->causal,
        have_init);
  }
  RACE_CU(cudaGetLastError());
  {
    RACE_LAUNCH("hard_normalize", s);
    hard::k_hard_normalize<TO><<<(unsigned)((rows * kD + 255) / 256), 256, 0, s>>>(
        num, cnt, out, (int64_t)rows);
  }
  RACE_CU(cudaGetLastError());
  return RACE_OK;
}

// Scratch: the caller's, or stream-ordered memory of our own.
struct Scratch {
  char* ptr = nullptr;
  bool owned = false;
  cudaStream_t s = nullptr;
  race_status_t acquire(const race_args_t* a, size_t need, cudaStream_t st) {
    s = st;
    if (need == 0) return RACE_OK;
    if (a->workspace) {
      if (a->workspace_bytes < need) return RACE_ERR_WORKSPACE;
      if ((reinterpret_cast<uintptr_t>(a->workspace) & (kAlign - 1)) != 0)
        return RACE_ERR_INVALID_ARG;
      ptr = static_cast<char*>(a->workspace);
      return RACE_OK;
    }
    void* p = nullptr;
    if (cudaMallocAsync(&p, need, st) != cudaSuccess) {
      cudaGetLastError();
      return RACE_ERR_WORKSPACE;
    }
    ptr = static_cast<char*>(p);
    owned = true;
    return RACE_OK;
  }
  ~Scratch() {
    if (owned) cudaFreeAsync(ptr, s);
  }
};

race_status_t forward_impl(const void* q, const void* k, const void* v, const float* W,
                           void* out, const race_args_t* a, cudaStream_t s,
                           const Carry* cy = nullptr) {
  race_status_t st = check_args(a);
  if (st != RACE_OK) return st;
  if (!q || !k || !v || !W || !out) return RACE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(W) || !aligned16(out) ||
      (a->den && !aligned16(a->den)))
    return RACE_ERR_INVALID_ARG;
  const bool tensor = use_tensor_path(a);
  if (a->impl == RACE_IMPL_TENSOR && !tensor) return RACE_ERR_UNSUPPORTED;
  Scratch sc;
  st = sc.acquire(a, workspace_bytes(a, false), s);
  if (st != RACE_OK) return st;
  if (tensor) {
    if (a->out_dtype == RACE_BF16)
      return tc_forward(a, q, k, v, W, static_cast<__nv_bfloat16*>(out), sc.ptr, s, cy);
    return tc_forward(a, q, k, v, W, static_cast<float*>(out), sc.ptr, s, cy);
  }
  if (a->dtype == RACE_BF16) {
    auto* qq = static_cast<const __nv_bfloat16*>(q);
    auto* kk = static_cast<const __nv_bfloat16*>(k);
    auto* vv = static_cast<const __nv_bfloat16*>(v);
    if (a->out_dtype == RACE_BF16)
      return simt_forward(a, qq, kk, vv, W, static_cast<__nv_bfloat16*>(out), sc.ptr, s, cy);
    return simt_forward(a, qq, kk, vv, W, static_cast<float*>(out), sc.ptr, s, cy);
  }
  auto* qq = static_cast<const float*>(q);
  auto* kk = static_cast<const float*>(k);
  auto* vv = static_cast<const float*>(v);
  if (a->out_dtype == RACE_BF16)
    return simt_forward(a, qq, kk, vv, W, static_cast<__nv_bfloat16*>(out), sc.ptr, s, cy);
  return simt_forward(a, qq, kk, vv, W, static_cast<float*>(out), sc.ptr, s, cy);
}

race_status_t backward_impl(const void* q, const void* k, const void* v, const float* W,
                            const void* out, const void* dout, void* dq, void* dk, void* dv,
                            float* dW, const race_args_t* a, cudaStream_t s) {
  race_status_t st = check_args(a);
  if (st != RACE_OK) return st;
  const void* ptrs[] = {q, k, v, W, out, dout, dq, dk, dv, dW};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return RACE_ERR_INVALID_ARG;
  if (a->den && !aligned16(a->den)) return RACE_ERR_INVALID_ARG;
  const bool tensor = use_tensor_backward(a);
  if (a->impl == RACE_IMPL_TENSOR && !tensor) return RACE_ERR_UNSUPPORTED;
  Scratch sc;
  st = sc.acquire(a, workspace_bytes(a, true), s);
  if (st != RACE_OK) return st;
  if (tensor) {
    auto* qq = static_cast<const __nv_bfloat16*>(q);
    auto* kk = static_cast<const __nv_bfloat16*>(k);
    auto* vv = static_cast<const __nv_bfloat16*>(v);
    auto* gg = static_cast<const __nv_bfloat16*>(dout);
#define RACE_TBWD(TO, TG)                                                                 \
  return tc_backward<TO, TG>(a, qq, kk, vv, W, static_cast<const TO*>(out), gg,          \
                             static_cast<TG*>(dq), static_cast<TG*>(dk), static_cast<TG*>(dv), \
                             dW, sc.ptr, s)
    if (a->out_dtype == RACE_BF16) {
      if (a->grad_dtype == RACE_BF16) RACE_TBWD(__nv_bfloat16, __nv_bfloat16);
      RACE_TBWD(__nv_bfloat16, float);
    }
    if (a->grad_dtype == RACE_BF16) RACE_TBWD(float, __nv_bfloat16);
    RACE_TBWD(float, float);
#undef RACE_TBWD
  }
#define RACE_BWD(T, TO, TG)                                                                \
  return simt_backward<T, TO, TG>(a, static_cast<const T*>(q), static_cast<const T*>(k),   \
                                  static_cast<const T*>(v), W, static_cast<const TO*>(out), \
                                  static_cast<const T*>(dout), static_cast<TG*>(dq),        \
                                  static_cast<TG*>(dk), static_cast<TG*>(dv), dW, sc.ptr, s)
#define RACE_BWD_G(T, TO)                                        \
  do {                                                           \
    if (a->grad_dtype == RACE_BF16) RACE_BWD(T, TO, __nv_bfloat16); \
    RACE_BWD(T, TO, float);                                      \
  } while (0)
  if (a->dtype == RACE_BF16) {
    if (a->out_dtype == RACE_BF16) RACE_BWD_G(__nv_bfloat16, __nv_bfloat16);
    RACE_BWD_G(__nv_bfloat16, float);
  }
  if (a->out_dtype == RACE_BF16) RACE_BWD_G(float, __nv_bfloat16);
  RACE_BWD_G(float, float);
#undef RACE_BWD_G
#undef RACE_BWD
}

// Result word of race_selftest_wait_timeout (1: every lane of the test kernel gave up).
__device__ int g_selftest_result = 0;

// ------------------------------------------------------------ allocation-free forward
// Scratch of race_forward_noalloc.  Some callers cannot allocate device memory at call
// time: a serving process that reserved all free HBM for its caches at start-up, or a
// latency-bound loop that must not enter an allocator (which can synchronise or grow
// its pool).  For them the scratch is this fixed array, part of the loaded module: it
// costs RACE_NOALLOC_SCRATCH_BYTES on every device the module is loaded on and is
// shared by all calls on that device, so overlapping calls race.
static __device__ __align__(256) char g_noalloc_scratch[RACE_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.  It is looked up on every
// call (a table look-up once the module is loaded there) rather than cached, so that a
// device reset or a different context on the same device cannot leave a stale address.
// The first look-up on a device may load the module there, which is why the first call
// belongs before any stream capture.
race_status_t noalloc_scratch(char** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p) {
    cudaGetLastError();
    return RACE_ERR_CUDA;
  }
  *out = static_cast<char*>(p);
  return RACE_OK;
}

}  // namespace
}  // namespace race

using namespace race;

extern "C" {

void race_args_init(race_args_t* a, int64_t N, int H, int d, int L, int P, float tau,
                    int causal) {
  if (!a) return;
  std::memset(a, 0, sizeof(*a));
  a->N = N;
  a->H = H;
  a->d = d;
  a->L = L;
  a->P = P;
  a->tau = tau;
  a->causal = causal;
  a->dtype = RACE_BF16;
  a->out_dtype = RACE_BF16;
  a->grad_dtype = RACE_BF16;
  a->impl = RACE_IMPL_AUTO;
}

race_status_t race_forward(const void* q, const void* k, const void* v, const float* W,
                           void* out, int64_t N, int H, int d, int L, int P, float tau,
                           int causal, race_stream_t stream) {
  NvtxRange r("race_forward");
  race_args_t a;
  race_args_init(&a, N, H, d, L, P, tau, causal);
  return forward_impl(q, k, v, W, out, &a, reinterpret_cast<cudaStream_t>(stream));
}

race_status_t race_backward(const void* q, const void* k, const void* v, const float* W,
                            const void* out, const void* dout, void* dq, void* dk,
                            void* dv, float* dW, int64_t N, int H, int d, int L, int P,
                            float tau, int causal, race_stream_t stream) {
  NvtxRange r("race_backward");
  race_args_t a;
  race_args_init(&a, N, H, d, L, P, tau, causal);
  return backward_impl(q, k, v, W, out, dout, dq, dk, dv, dW, &a,
                       reinterpret_cast<cudaStream_t>(stream));
}

race_status_t race_forward_ex(const void* q, const void* k, const void* v, const float* W,
                              void* out, const race_args_t* a, race_stream_t stream) {
  NvtxRange r("race_forward_ex");
  return forward_impl(q, k, v, W, out, a, reinterpret_cast<cudaStream_t>(stream));
}

race_status_t race_backward_ex(const void* q, const void* k, const void* v,
                               const float* W, const void* out, const void* dout, void* dq,
                               void* dk, void* dv, float* dW, const race_args_t* a,
                               race_stream_t stream) {
  NvtxRange r("race_backward_ex");
  return backward_impl(q, k, v, W, out, dout, dq, dk, dv, dW, a,
                       reinterpret_cast<cudaStream_t>(stream));
}

race_status_t race_forward_noalloc(const void* q, const void* k, const void* v,
                                   const float* W, void* out, const race_args_t* a,
                                   race_stream_t stream) {
  NvtxRange r("race_forward_noalloc");
  if (!a) return RACE_ERR_INVALID_ARG;
  race_status_t st = check_args(a);
  if (st != RACE_OK) return st;
  if (workspace_bytes(a, false) > RACE_NOALLOC_SCRATCH_BYTES) return RACE_ERR_SCRATCH_LIMIT;
  char* ws = nullptr;
  st = noalloc_scratch(&ws);
  if (st != RACE_OK) return st;
  // The forward clears its accumulators itself (every path memsets or fully writes
  // the scratch it reads), so the array needs no clearing between calls.
  race_args_t b = *a;
  b.workspace = ws;
  b.workspace_bytes = RACE_NOALLOC_SCRATCH_BYTES;
  return forward_impl(q, k, v, W, out, &b, reinterpret_cast<cudaStream_t>(stream));
}

race_status_t race_forward_stream(const void* q, const void* k, const void* v,
                                  const float* W, void* out, const float* state_in,
                                  float* state_out, const race_args_t* a,
                                  race_stream_t stream) {
  NvtxRange r("race_forward_stream");
  if ((state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)))
    return RACE_ERR_INVALID_ARG;
  Carry cy;
  cy.in = state_in;
  cy.out = state_out;
  cy.on = true;
  return forward_impl(q, k, v, W, out, a, reinterpret_cast<cudaStream_t>(stream), &cy);
}

race_status_t race_hard_workspace_size(const race_args_t* a, size_t* bytes) {
  if (bytes) *bytes = 0;
  if (!bytes) return RACE_ERR_INVALID_ARG;
  race_status_t st = check_args(a);
  if (st != RACE_OK) return st;
  *bytes = hard_plan(a).bytes;
  return RACE_OK;
}

race_status_t race_hard_forward(const void* q, const void* k, const void* v, const float* W,
                                void* out, int* counts, const race_args_t* a,
                                race_stream_t stream) {
  NvtxRange r("race_hard_forward");
  race_status_t st = check_args(a);
  if (st != RACE_OK) return st;
  const void* ptrs[] = {q, k, v, W, out};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return RACE_ERR_INVALID_ARG;
  if (counts && !aligned16(counts)) return RACE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Scratch sc;
  st = sc.acquire(a, hard_plan(a).bytes, s);
  if (st != RACE_OK) return st;
#define RACE_HARD(T, TO)                                                                    \
  return hard_forward<T, TO>(a, static_cast<const T*>(q), static_cast<const T*>(k),       \
                             static_cast<const T*>(v), W, static_cast<TO*>(out), counts,  \
                             sc.ptr, s)
  if (a->dtype == RACE_BF16) {
    if (a->out_dtype == RACE_BF16) RACE_HARD(__nv_bfloat16, __nv_bfloat16);
    RACE_HARD(__nv_bfloat16, float);
  }
  if (a->out_dtype == RACE_BF16) RACE_HARD(float, __nv_bfloat16);
  RACE_HARD(float, float);
#undef RACE_HARD
}

race_status_t race_hard_hash(const void* x, const float* W, uint8_t* ids, const race_args_t* a,
                             race_stream_t stream) {
  race_status_t st = check_args(a);
  if (st != RACE_OK) return st;
  if (!x || !W || !ids || !aligned16(x) || !aligned16(W)) return RACE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (a->dtype == RACE_BF16)
    return hard_ids<__nv_bfloat16>(a, static_cast<const __nv_bfloat16*>(x), W, ids, s);
  return hard_ids<float>(a, static_cast<const float*>(x), W, ids, s);
}

race_status_t race_workspace_size(const race_args_t* a, int backward, size_t* bytes) {
  if (bytes) *bytes = 0;
  if (!bytes) return RACE_ERR_INVALID_ARG;
  race_status_t st = check_args(a);
  if (st != RACE_OK) return st;
  if (a->impl == RACE_IMPL_TENSOR && (backward || !use_tensor_path(a)))
    return RACE_ERR_UNSUPPORTED;
  *bytes = workspace_bytes(a, backward != 0);
  return RACE_OK;
}

race_status_t race_hash(const void* x, const float* W, void* phi, const race_args_t* a,
                        race_stream_t stream) {
  race_status_t st = check_args(a);
  if (st != RACE_OK) return st;
  if (!x || !W || !phi || !aligned16(x) || !aligned16(W) || !aligned16(phi))
    return RACE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Dims dm = dims_of(a);
  simt::Layout ly(dm.R, dm.P);
  dim3 grid((unsigned)((a->N + simt::TT - 1) / simt::TT), a->H);
#define RACE_HASH(T, TO)                                                            \
  do {                                                                              \
    RACE_CU(set_smem(simt::k_hash<T, TO>, ly.bytes()));                             \
    RACE_LAUNCH("simt_hash", s);                                                    \
    simt::k_hash<T, TO><<<grid, simt::NT, ly.bytes(), s>>>(                         \
        static_cast<const T*>(x), W, static_cast<TO*>(phi), dm);                    \
  } while (0)
  if (a->dtype == RACE_BF16) {
    if (a->out_dtype == RACE_BF16) RACE_HASH(__nv_bfloat16, __nv_bfloat16);
    else RACE_HASH(__nv_bfloat16, float);
  } else {
    if (a->out_dtype == RACE_BF16) RACE_HASH(float, __nv_bfloat16);
    else RACE_HASH(float, float);
  }
#undef RACE_HASH
  RACE_CU(cudaGetLastError());
  return RACE_OK;
}

race_status_t race_selftest_wait_timeout(int64_t limit_cycles, int* timed_out,
                                         race_stream_t stream) {
  if (timed_out) *timed_out = 0;
  if (limit_cycles < 1 || limit_cycles > tc::kWaitCycles) return RACE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* res = nullptr;
  RACE_CU(cudaGetSymbolAddress(reinterpret_cast<void**>(&res), g_selftest_result));
  RACE_CU(cudaMemsetAsync(res, 0, sizeof(int), s));
  {
    RACE_LAUNCH("selftest_wait_timeout", s);
    tc::k_selftest_wait_timeout<<<1, 32, 0, s>>>((long long)limit_cycles, res);
  }
  RACE_CU(cudaGetLastError());
  int v = 0;
  RACE_CU(cudaMemcpyAsync(&v, res, sizeof(int), cudaMemcpyDeviceToHost, s));
  RACE_CU(cudaStreamSynchronize(s));
  if (timed_out) *timed_out = v;
  return RACE_OK;
}

race_status_t race_device_status(race_stream_t stream, uint32_t* flags) {
  if (flags) *flags = 0;
  RACE_CU(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  uint32_t v = 0, zero = 0;
  RACE_CU(cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)));
  RACE_CU(cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)));
  if (flags) *flags = v;
  return v ? RACE_ERR_DEVICE_STATUS : RACE_OK;
}

const char* race_status_string(race_status_t s) {
  switch (s) {
    case RACE_OK: return "RACE_OK";
    case RACE_ERR_INVALID_ARG: return "RACE_ERR_INVALID_ARG: invalid argument";
    case RACE_ERR_UNSUPPORTED: return "RACE_ERR_UNSUPPORTED: unsupported configuration";
    case RACE_ERR_WORKSPACE: return "RACE_ERR_WORKSPACE: scratch too small or allocation failed";
    case RACE_ERR_CUDA: return "RACE_ERR_CUDA: CUDA call or launch failed";
    case RACE_ERR_DEVICE_STATUS: return "RACE_ERR_DEVICE_STATUS: a kernel raised the device status flag";
    case RACE_ERR_SCRATCH_LIMIT:
      return "RACE_ERR_SCRATCH_LIMIT: problem needs more scratch than the fixed "
             "RACE_NOALLOC_SCRATCH_BYTES array of race_forward_noalloc";
  }
  return "unknown race_status_t";
}

int race_version(void) { return 100; }

race_status_t race_timing_enable(int on) {
  std::lock_guard<std::mutex> lk(launches::g_mu);
  launches::drain();
  launches::g_timers.clear();
  launches::g_timing = on != 0;
  return RACE_OK;
}

race_status_t race_timing_report(int i, const char** name, double* total_ms,
                                 int64_t* count) {
  std::lock_guard<std::mutex> lk(launches::g_mu);
  launches::drain();
  if (i < 0 || i >= (int)launches::g_timers.size()) return RACE_ERR_INVALID_ARG;
  const auto& t = launches::g_timers[i];
  if (name) *name = t.name.c_str();
  if (total_ms) *total_ms = t.ms;
  if (count) *count = t.n;
  return RACE_OK;
}

int64_t race_launch_count(void) { return launches::g_count.load(); }

#ifdef RACE_SWEEP_TRACE
// Copies the sweep timeline (see tc_sweep.cuh) to host memory `dst`; returns the
// number of 64-bit stamps.
int race_sweep_trace_read(unsigned long long* dst) {
  cudaDeviceSynchronize();
  cudaMemcpyFromSymbol(dst, tc::g_sweep_trace, sizeof(tc::g_sweep_trace));
  return 2 * tc::kTraceChunks * tc::kTraceEvents;
}
#endif

}  // extern "C"
