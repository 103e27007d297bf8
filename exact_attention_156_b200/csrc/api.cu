// api.cu - the C ABI declared in include/attn.h: argument validation, launch
// planning (tile shapes per head_dim, grids), TMA descriptor encoding and
// kernel launches.  Nothing here computes attention; every step of the path
// runs in the kernels of fwd_sm100.cuh and bwd_sm100.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <math.h>
#include <initializer_list>
#include <mutex>
#include <stdint.h>
#include <string.h>
#include <type_traits>

#include "../../include/attn.h"
#include "bwd256_sm100.cuh"
#include "bwd_sm100.cuh"
#include "decode_sm100.cuh"
#include "fwd256_sm100.cuh"
#include "fwd_sm100.cuh"
#include "padded.cuh"

using namespace attn156;

namespace {

// Device error word written by timed-out waits (and by the alignment guard).
__device__ uint32_t g_attn_err = 0;

constexpr uint64_t kTimeoutNs = 1000000000ull;  // 1 s per device-side wait
// Block order: the operands that the CTAs of a chunk of heads stream (K/V in
// the forward; Q, dO and the dQ accumulator in the backward) may take this many
// bytes, about half the 126 MB L2.
constexpr double kOrderChunkBytes = 64.0 * 1024 * 1024;
int order_chunk(double bytes_per_unit, int units) {
  const double c = bytes_per_unit > 0 ? kOrderChunkBytes / bytes_per_unit : units;
  return c >= units ? units : (c < 1.0 ? 1 : int(c));
}
constexpr int kMaxDevices = 64;

struct DeviceState {
  bool init = false;
  bool arch_ok = false;
  uint32_t* err = nullptr;
  int num_sms = 0;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <typename K>
int regs_of(K kernel) {
  cudaFuncAttributes a;
  if (cudaFuncGetAttributes(&a, kernel) != cudaSuccess) return -1;
  return a.numRegs;
}

// One-time per-device set-up: architecture check, error-word address, kernel attributes.
attn_status device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_DEVICE;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.init) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return ATTN_ERR_DEVICE;
    cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev);
    s.arch_ok = (major == 10 && minor == 0);
    if (s.arch_ok) {
      if (cudaGetSymbolAddress(reinterpret_cast<void**>(&s.err), g_attn_err) != cudaSuccess)
        return ATTN_ERR_LAUNCH;
      // The warp-specialised kernels hand registers between warpgroups with
      // setmaxnreg; the split is sized for exactly kLaunchRegs per thread at
      // launch.  Refuse to launch a build whose allocation differs.
      bool ok = true;
      auto prepare = [&](auto d, auto e) {
        constexpr int D = decltype(d)::value;
        using E = decltype(e);
        auto both = [&](auto v) {
          constexpr bool kV = decltype(v)::value;
          ok = ok &&
               set_smem(fwd::attn_fwd_kernel<D, E, kV>, fwd::Cfg<D>::kSmemBytes) == cudaSuccess &&
               set_smem(bwd::attn_bwd_main_kernel<D, E, kV>, bwd::Cfg<D>::kSmemBytes) ==
                   cudaSuccess &&
               regs_of(fwd::attn_fwd_kernel<D, E, kV>) == fwd::kLaunchRegs &&
               regs_of(bwd::attn_bwd_main_kernel<D, E, kV>) == bwd::kLaunchRegs;
        };
        both(std::false_type{});  // (B, S, H, D) batches
        both(std::true_type{});   // packed variable-length batches
        ok = ok &&
             set_smem(dec::attn_decode_kernel<D, E>, dec::Cfg<D>::kSmemBytes) == cudaSuccess &&
             set_smem(fwd256::attn_fwd_d256_kernel<E>, fwd256::Cfg::kSmemBytes) == cudaSuccess;
        ok = ok && set_smem(dec::t16::attn_decode_t16_kernel<D, E>,
                            dec::t16::Cfg<D>::kSmemBytes) == cudaSuccess;
      };
      ok = ok &&
           set_smem(bwd256::attn_bwd_d256_kernel<ElemBF16>, bwd256::Cfg::kSmemBytes) ==
               cudaSuccess &&
           set_smem(bwd256::attn_bwd_d256_kernel<ElemF16>, bwd256::Cfg::kSmemBytes) == cudaSuccess;
      prepare(std::integral_constant<int, 64>{}, ElemBF16{});
      prepare(std::integral_constant<int, 128>{}, ElemBF16{});
      prepare(std::integral_constant<int, 64>{}, ElemF16{});
      prepare(std::integral_constant<int, 128>{}, ElemF16{});
      if (!ok) return ATTN_ERR_LAUNCH;
      if (g_encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
          return ATTN_ERR_LAUNCH;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
      }
    }
    s.init = true;
  }
  if (!s.arch_ok) return ATTN_ERR_ARCH;
  *out = &s;
  return ATTN_OK;
}

// A pointer must be device (or managed) memory visible from the current device.
bool on_current_device(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  int dev = -1;
  cudaGetDevice(&dev);
  if (a.type == cudaMemoryTypeDevice) return a.device == dev;
  if (a.type == cudaMemoryTypeManaged) return true;
  return false;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

attn_status check_common(int B, int Sq, int Sk, int H, int D, float scale, int win_left,
                         int win_right, int Hk = -1, bool allow_d256 = false) {
  if (Hk < 0) Hk = H;
  if (B < 1 || Sq < 1 || Sk < 1 || H < 1) return ATTN_ERR_SHAPE;
  if (B > 65535 || H > 65535) return ATTN_ERR_SHAPE;
  if (Hk < 1 || Hk > H || H % Hk != 0) return ATTN_ERR_SHAPE;
  if (D != 64 && D != 128 && !(allow_d256 && D == 256)) return ATTN_ERR_HEADDIM;
  if ((long long)B * Sq * H * D >= (1ll << 31) || (long long)B * Sk * Hk * D >= (1ll << 31))
    return ATTN_ERR_SHAPE;
  if (!(scale > 0.f) || !isfinite(scale)) return ATTN_ERR_SHAPE;
  if (win_left < -1 || win_right < -1) return ATTN_ERR_WINDOW;
  return ATTN_OK;
}

// TMA element type of a kernel element format.
template <class E>
constexpr CUtensorMapDataType tmap_type() {
  return std::is_same<E, ElemF16>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                          : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
}

// Encoded tensor maps, cached per (device, base address, element type, rank,
// extents, strides, box): a map is a pure function of these, so a cached one
// stays valid for as long as the same arguments come back (a buffer freed and
// reallocated at the same address with the same shape gets the same map).
// Small and round-robin: one call needs at most eight maps.  Every map in this
// library uses 128-byte swizzle, no interleave, 256-byte L2 promotion, zero
// fill out of bounds and unit element strides.
struct MapKey {
  int dev, rank;
  CUtensorMapDataType dtype;
  const void* base;
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4];
  bool operator==(const MapKey& o) const {
    if (dev != o.dev || rank != o.rank || dtype != o.dtype || base != o.base) return false;
    for (int i = 0; i < rank; ++i)
      if (dims[i] != o.dims[i] || box[i] != o.box[i]) return false;
    for (int i = 0; i + 1 < rank; ++i)
      if (strides[i] != o.strides[i]) return false;
    return true;
  }
};
constexpr int kMapCacheSize = 64;
struct MapCache {
  MapKey key[kMapCacheSize];
  alignas(64) CUtensorMap map[kMapCacheSize];
  bool used[kMapCacheSize] = {};
  int next = 0;
};
MapCache g_maps;
std::mutex g_maps_mu;

attn_status encode_cached(CUtensorMap* out, CUtensorMapDataType dtype, int rank, const void* base,
                          const cuuint64_t* dims, const cuuint64_t* strides,
                          const cuuint32_t* box) {
  MapKey k{};
  if (cudaGetDevice(&k.dev) != cudaSuccess) return ATTN_ERR_DEVICE;
  k.rank = rank;
  k.dtype = dtype;
  k.base = base;
  for (int i = 0; i < rank; ++i) {
    k.dims[i] = dims[i];
    k.box[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) k.strides[i] = strides[i];
  std::lock_guard<std::mutex> lock(g_maps_mu);
  for (int i = 0; i < kMapCacheSize; ++i)
    if (g_maps.used[i] && g_maps.key[i] == k) {
      *out = g_maps.map[i];
      return ATTN_OK;
    }
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r =
      g_encode(out, dtype, cuuint32_t(rank), const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return ATTN_ERR_LAUNCH;
  const int slot = g_maps.next;
  g_maps.next = (slot + 1) % kMapCacheSize;
  g_maps.key[slot] = k;
  g_maps.map[slot] = *out;
  g_maps.used[slot] = true;
  return ATTN_OK;
}

// 4-D map over a (B, S, H, D) tensor of 16-bit elements, box = 64 x 1 x rows x 1
// (rows = 128 unless given), 128-byte swizzle.
attn_status make_map(CUtensorMap* map, const void* base, int B, int S, int H, int D,
                     CUtensorMapDataType dtype, int box_rows = 128) {
  const cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(S), cuuint64_t(B)};
  const cuuint64_t strides[3] = {cuuint64_t(D) * 2, cuuint64_t(H) * D * 2,
                                 cuuint64_t(S) * H * D * 2};
  const cuuint32_t box[4] = {64, 1, cuuint32_t(box_rows), 1};
  return encode_cached(map, dtype, 4, base, dims, strides, box);
}

// 2-D fp32 map over the dQ accumulator [rows][D], box = 32 x 128, 128-byte swizzle
// (the layout the backward's drain warps stage a dQ tile in).
attn_status make_dq_map(CUtensorMap* map, const float* base, long long rows, int D) {
  const cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(D) * 4};
  const cuuint32_t box[2] = {32, 128};
  return encode_cached(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box);
}

int sq_pad(int Sq) { return ((Sq + 127) / 128) * 128; }

size_t workspace_bytes(int B, int Sq, int H, int D) {
  const size_t rows = size_t(B) * H * sq_pad(Sq);
  return rows * D * 4 + rows * 4 * 2;
}

template <int D, class E>
attn_status launch_fwd(const DeviceState& st, const void* q, const void* k, const void* v, void* o,
                       float* lse, int B, int Sq, int Sk, int H, int Hk, float scale, int causal,
                       int win_left, int win_right, cudaStream_t stream) {
  constexpr CUtensorMapDataType dt = tmap_type<E>();
  alignas(64) CUtensorMap mq, mk, mv;
  if (make_map(&mq, q, B, Sq, H, D, dt) != ATTN_OK || make_map(&mk, k, B, Sk, Hk, D, dt) != ATTN_OK ||
      make_map(&mv, v, B, Sk, Hk, D, dt) != ATTN_OK)
    return ATTN_ERR_LAUNCH;
  fwd::Params p;
  p.o = static_cast<uint16_t*>(o);
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Hk = Hk;
  p.Sq = Sq;
  p.Sk = Sk;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.win_left = win_left;
  p.win_right = win_right;
  p.cu_q = nullptr;
  p.cu_k = nullptr;
  p.total_q = 0;
  p.total_k = 0;
  p.num_mblocks = (Sq + fwd::NQ * fwd::BM - 1) / (fwd::NQ * fwd::BM);
  p.compact = 0;
  // Block order: pair-major within chunks of heads whose K and V fit in L2
  // together (K/V bytes per query head: a K/V head's, shared by H / Hk heads)
  p.order_chunk = order_chunk(2.0 * double(Sk) * D * 2.0 * Hk / H, H * B);
  p.err = st.err;
  p.timeout_ns = kTimeoutNs;
  dim3 grid(p.num_mblocks, H, B);
  fwd::attn_fwd_kernel<D, E, false><<<grid, fwd::kThreads, fwd::Cfg<D>::kSmemBytes, stream>>>(mq, mk, mv,
                                                                                       p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

// head_dim 256 forward: one 128-row query tile per CTA, 128-key K/V tiles.
template <class E>
attn_status launch_fwd_d256(const DeviceState& st, const void* q, const void* k, const void* v,
                            void* o, float* lse, int B, int Sq, int Sk, int H, int Hk, float scale,
                            int causal, int win_left, int win_right, cudaStream_t stream) {
  constexpr CUtensorMapDataType dt = tmap_type<E>();
  alignas(64) CUtensorMap mq, mk, mv;
  if (make_map(&mq, q, B, Sq, H, 256, dt, fwd256::BM) != ATTN_OK ||
      make_map(&mk, k, B, Sk, Hk, 256, dt, fwd256::BN) != ATTN_OK ||
      make_map(&mv, v, B, Sk, Hk, 256, dt, fwd256::BN) != ATTN_OK)
    return ATTN_ERR_LAUNCH;
  fwd256::Params p;
  p.o = static_cast<uint16_t*>(o);
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Sq = Sq;
  p.Sk = Sk;
  p.Hk = Hk;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.win_left = win_left;
  p.win_right = win_right;
  p.num_mblocks = (Sq + fwd256::BM - 1) / fwd256::BM;
  p.order_chunk = order_chunk(2.0 * double(Sk) * 256 * 2.0 * Hk / H, H * B);
  p.err = st.err;
  p.timeout_ns = kTimeoutNs;
  fwd256::attn_fwd_d256_kernel<E><<<dim3(p.num_mblocks, H, B), fwd256::kThreads,
                                    fwd256::Cfg::kSmemBytes, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

struct Workspace {
  float* dq_acc;  // [B*H][Sq_pad][D]
  float* nlse2;   // [B*H][Sq_pad] -LSE * log2(e)
  float* ndelta;  // [B*H][Sq_pad] -rowsum(dO * O)
  int Sq_pad;
};

Workspace carve(void* workspace, int B, int Sq, int H, int D) {
  Workspace w;
  w.Sq_pad = sq_pad(Sq);
  const size_t rows = size_t(B) * H * w.Sq_pad;
  w.dq_acc = static_cast<float*>(workspace);
  w.nlse2 = w.dq_acc + rows * D;
  w.ndelta = w.nlse2 + rows;
  return w;
}

template <int D, class E>
attn_status launch_bwd_pre(const void* o, const void* dout, const float* lse, int B, int Sq,
                           int H, const Workspace& w, cudaStream_t stream) {
  const long long rows = (long long)B * H * w.Sq_pad;
  const long long per_block = 8LL * bwd::kPreRows;  // 8 warps of kPreRows rows
  const unsigned blocks = unsigned((rows + per_block - 1) / per_block);
  // head_dim 256 writes dQ rows whole (no reduce-add), so its accumulator needs no clearing
  bwd::attn_bwd_pre_kernel<D, E><<<blocks, 256, 0, stream>>>(
      static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), lse, w.nlse2,
      w.ndelta, D == 256 ? nullptr : w.dq_acc, B, H, Sq, w.Sq_pad);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

template <int D, class E>
attn_status launch_bwd_main(const DeviceState& st, const void* q, const void* k, const void* v,
                            const void* dout, void* dk, void* dv, int B, int Sq, int Sk, int H,
                            int Hk, float scale, int causal, int win_left, int win_right,
                            const Workspace& w, cudaStream_t stream) {
  constexpr CUtensorMapDataType dt = tmap_type<E>();
  alignas(64) CUtensorMap mq, mk, mv, mdo, mdq;
  if (make_map(&mq, q, B, Sq, H, D, dt) != ATTN_OK || make_map(&mk, k, B, Sk, Hk, D, dt) != ATTN_OK ||
      make_map(&mv, v, B, Sk, Hk, D, dt) != ATTN_OK ||
      make_map(&mdo, dout, B, Sq, H, D, dt) != ATTN_OK ||
      make_dq_map(&mdq, w.dq_acc, (long long)B * H * w.Sq_pad, D) != ATTN_OK)
    return ATTN_ERR_LAUNCH;
  bwd::Params p;
  p.dk = static_cast<uint16_t*>(dk);
  p.dv = static_cast<uint16_t*>(dv);
  p.nlse2 = w.nlse2;
  p.ndelta = w.ndelta;
  p.dq_acc = w.dq_acc;
  p.B = B;
  p.H = H;
  p.Sq = Sq;
  p.Sk = Sk;
  p.Sq_pad = w.Sq_pad;
  p.cu_q = nullptr;
  p.cu_k = nullptr;
  p.total_q = 0;
  p.total_k = 0;
  p.R = 0;
  p.compact = 0;
  // Block order (as in the forward): tile-major within chunks of K/V heads
  // whose streamed operands (Q, dO and the fp32 dQ accumulator of the H / Hk
  // query heads each serves) fit in L2 together.
  p.order_chunk = order_chunk(double(H / Hk) * double(Sq) * D * (2.0 + 2.0 + 4.0), Hk * B);
  p.Hk = Hk;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.win_left = win_left;
  p.win_right = win_right;
  p.err = st.err;
  p.timeout_ns = kTimeoutNs;
  dim3 grid((Sk + bwd::BN - 1) / bwd::BN, Hk, B);
  bwd::attn_bwd_main_kernel<D, E, false>
      <<<grid, bwd::kThreads, bwd::Cfg<D>::kSmemBytes, stream>>>(mq, mk, mv, mdo, mdq, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

// head_dim 256 backward: one launch of dK, dV and dQ tiles (see bwd256_sm100.cuh).
template <class E>
attn_status launch_bwd_main_d256(const DeviceState& st, const void* q, const void* k,
                                 const void* v, const void* dout, void* dk, void* dv, int B,
                                 int Sq, int Sk, int H, int Hk, float scale, int causal,
                                 int win_left, int win_right, const Workspace& w,
                                 cudaStream_t stream) {
  constexpr CUtensorMapDataType dt = tmap_type<E>();
  alignas(64) CUtensorMap q128, k128, v128, do128, q64, k64, v64, do64;
  if (make_map(&q128, q, B, Sq, H, 256, dt, 128) != ATTN_OK ||
      make_map(&k128, k, B, Sk, Hk, 256, dt, 128) != ATTN_OK ||
      make_map(&v128, v, B, Sk, Hk, 256, dt, 128) != ATTN_OK ||
      make_map(&do128, dout, B, Sq, H, 256, dt, 128) != ATTN_OK ||
      make_map(&q64, q, B, Sq, H, 256, dt, 64) != ATTN_OK ||
      make_map(&k64, k, B, Sk, Hk, 256, dt, 64) != ATTN_OK ||
      make_map(&v64, v, B, Sk, Hk, 256, dt, 64) != ATTN_OK ||
      make_map(&do64, dout, B, Sq, H, 256, dt, 64) != ATTN_OK)
    return ATTN_ERR_LAUNCH;
  bwd256::Params p;
  p.dk = static_cast<uint16_t*>(dk);
  p.dv = static_cast<uint16_t*>(dv);
  p.dq_acc = w.dq_acc;
  p.nlse2 = w.nlse2;
  p.ndelta = w.ndelta;
  p.B = B;
  p.H = H;
  p.Hk = Hk;
  p.Sq = Sq;
  p.Sk = Sk;
  p.Sq_pad = w.Sq_pad;
  p.n_ktiles = (Sk + bwd256::BR - 1) / bwd256::BR;
  p.n_qtiles = (Sq + bwd256::BR - 1) / bwd256::BR;
  // chunked block order over the heads (Q, dO and the float32 dQ rows of a head)
  p.order_chunk = order_chunk(double(Sq) * 256 * (2.0 + 2.0 + 4.0), H * B);
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.win_left = win_left;
  p.win_right = win_right;
  p.err = st.err;
  p.timeout_ns = kTimeoutNs;
  const dim3 grid(2 * p.n_ktiles + p.n_qtiles, H, B);
  bwd256::attn_bwd_d256_kernel<E><<<grid, bwd256::kThreads, bwd256::Cfg::kSmemBytes, stream>>>(
      q128, k128, v128, do128, q64, k64, v64, do64, p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

template <int D, class E>
attn_status launch_bwd_dq(void* dq, int B, int Sq, int H, float scale, const Workspace& w,
                          cudaStream_t stream) {
  const long long total = (long long)B * Sq * H * (D / 8);
  const unsigned blocks = unsigned((total + 255) / 256);
  bwd::attn_bwd_dq_kernel<D, E><<<blocks, 256, 0, stream>>>(
      w.dq_acc, static_cast<uint16_t*>(dq), B, H, Sq, w.Sq_pad, scale);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

// Calls f(integral_constant<int, D>, element format) for the (head_dim, dtype)
// of a call; both were validated before.
template <class F>
attn_status dispatch(int D, int dtype, F&& f) {
  if (dtype == ATTN_DTYPE_F16)
    return D == 64 ? f(std::integral_constant<int, 64>{}, ElemF16{})
                   : f(std::integral_constant<int, 128>{}, ElemF16{});
  return D == 64 ? f(std::integral_constant<int, 64>{}, ElemBF16{})
                 : f(std::integral_constant<int, 128>{}, ElemBF16{});
}

// As dispatch, with head_dim 256 too (the entry points whose kernels have a
// head_dim 256 form: the forward and the backward stages).
template <class F>
attn_status dispatch_d256(int D, int dtype, F&& f) {
  if (D == 256)
    return dtype == ATTN_DTYPE_F16 ? f(std::integral_constant<int, 256>{}, ElemF16{})
                                   : f(std::integral_constant<int, 256>{}, ElemBF16{});
  return dispatch(D, dtype, f);
}

// The backward's main stage for any supported head_dim.
template <int D, class E>
attn_status launch_bwd_main_any(const DeviceState& st, const void* q, const void* k,
                                const void* v, const void* dout, void* dk, void* dv, int B,
                                int Sq, int Sk, int H, int Hk, float scale, int causal,
                                int win_left, int win_right, const Workspace& w,
                                cudaStream_t cs) {
  if constexpr (D == 256)
    return launch_bwd_main_d256<E>(st, q, k, v, dout, dk, dv, B, Sq, Sk, H, Hk, scale, causal,
                                   win_left, win_right, w, cs);
  else
    return launch_bwd_main<D, E>(st, q, k, v, dout, dk, dv, B, Sq, Sk, H, Hk, scale, causal,
                                 win_left, win_right, w, cs);
}

attn_status check_dtype(int dtype) {
  return (dtype == ATTN_DTYPE_BF16 || dtype == ATTN_DTYPE_F16) ? ATTN_OK : ATTN_ERR_DTYPE;
}

// The three backward stages on one stream through workspace `w`.
attn_status run_backward(const DeviceState& st, const void* q, const void* k, const void* v,
                         const void* o, const void* dout, const float* lse, void* dq, void* dk,
                         void* dv, int B, int Sq, int Sk, int H, int Hk, int D, int dtype,
                         float scale, int causal, int win_left, int win_right, const Workspace& w,
                         cudaStream_t cs) {
  return dispatch_d256(D, dtype, [&](auto d, auto e) {
    constexpr int DD = decltype(d)::value;
    using E = decltype(e);
    attn_status s = launch_bwd_pre<DD, E>(o, dout, lse, B, Sq, H, w, cs);
    if (s == ATTN_OK)
      s = launch_bwd_main_any<DD, E>(st, q, k, v, dout, dk, dv, B, Sq, Sk, H, Hk, scale, causal,
                                     win_left, win_right, w, cs);
    if (s == ATTN_OK) s = launch_bwd_dq<DD, E>(dq, B, Sq, H, scale, w, cs);
    return s;
  });
}

// ---------------------------------------------------------------------------
// Packed variable-length batches
// ---------------------------------------------------------------------------
struct Varlen {
  const int* cu_q;  // [B + 1] device
  const int* cu_k;
  int total_q, total_k;
  int max_q, max_k;  // largest sequence lengths (the grid covers these)
};

// Rows per query head of the varlen row values and dQ accumulator: every
// sequence's block starts on a multiple of 4 rows and has 128 spare rows
// (the kernels' rv_start), so total_q + 132 B rows rounded up to 4 suffice.
long long varlen_rows(int B, int total_q) {
  return ((long long)total_q + 132ll * B + 3) & ~3ll;
}

size_t varlen_workspace_bytes(int B, int total_q, int H, int D) {
  const size_t rows = size_t(H) * size_t(varlen_rows(B, total_q));
  return rows * D * 4 + rows * 4 * 2;
}

attn_status check_varlen(int B, int total_q, int total_k, int max_q, int max_k, int H, int Hk,
                         int D, float scale, int win_left, int win_right) {
  if (B < 1 || B > 65535 || total_q < 1 || total_k < 1 || H < 1 || H > 65535)
    return ATTN_ERR_SHAPE;
  if (max_q < 1 || max_k < 1 || max_q > total_q || max_k > total_k) return ATTN_ERR_SHAPE;
  if (Hk < 1 || Hk > H || H % Hk != 0) return ATTN_ERR_SHAPE;
  if (D != 64 && D != 128) return ATTN_ERR_HEADDIM;
  if ((long long)total_q * H * D >= (1ll << 31) || (long long)total_k * Hk * D >= (1ll << 31) ||
      varlen_rows(B, total_q) * H * D >= (1ll << 31))
    return ATTN_ERR_SHAPE;
  if (!(scale > 0.f) || !isfinite(scale)) return ATTN_ERR_SHAPE;
  if (win_left < -1 || win_right < -1) return ATTN_ERR_WINDOW;
  return ATTN_OK;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

template <int D, class E>
attn_status launch_fwd_varlen(const DeviceState& st, const void* q, const void* k, const void* v,
                              void* o, float* lse, const Varlen& vl, int B, int H, int Hk,
                              float scale, int causal, int win_left, int win_right,
                              cudaStream_t stream) {
  constexpr CUtensorMapDataType dt = tmap_type<E>();
  alignas(64) CUtensorMap mq, mk, mv;
  if (make_map(&mq, q, 1, vl.total_q, H, D, dt) != ATTN_OK ||
      make_map(&mk, k, 1, vl.total_k, Hk, D, dt) != ATTN_OK ||
      make_map(&mv, v, 1, vl.total_k, Hk, D, dt) != ATTN_OK)
    return ATTN_ERR_LAUNCH;
  fwd::Params p;
  p.o = static_cast<uint16_t*>(o);
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Hk = Hk;
  p.Sq = vl.max_q;
  p.Sk = vl.max_k;
  p.cu_q = vl.cu_q;
  p.cu_k = vl.cu_k;
  p.total_q = vl.total_q;
  p.total_k = vl.total_k;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.win_left = win_left;
  p.win_right = win_right;
  p.num_mblocks = (vl.max_q + fwd::NQ * fwd::BM - 1) / (fwd::NQ * fwd::BM);
  p.err = st.err;
  p.timeout_ns = kTimeoutNs;
  // Up to kCompactMaxB sequences: one CTA per query-tile pair that has work
  // (at most ceil(total_q / 256) + B of them); otherwise the longest sequence's
  // pair count for every sequence.
  p.compact = B <= kCompactMaxB ? 1 : 0;
  // chunked block order over the heads (a head's K/V: every sequence's rows)
  p.order_chunk = order_chunk(2.0 * double(vl.total_k) * D * 2.0 * Hk / H,
                              p.compact ? H : H * B);
  const int rows = fwd::NQ * fwd::BM;
  dim3 grid = p.compact ? dim3((vl.total_q + rows - 1) / rows + B, H, 1)
                        : dim3(p.num_mblocks, H, B);
  fwd::attn_fwd_kernel<D, E, true><<<grid, fwd::kThreads, fwd::Cfg<D>::kSmemBytes, stream>>>(mq, mk, mv,
                                                                                       p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

template <int D, class E>
attn_status run_backward_varlen(const DeviceState& st, const void* q, const void* k,
                                const void* v, const void* o, const void* dout, const float* lse,
                                void* dq, void* dk, void* dv, const Varlen& vl, int B, int H,
                                int Hk, float scale, int causal, int win_left, int win_right,
                                void* workspace, cudaStream_t stream) {
  constexpr CUtensorMapDataType dt = tmap_type<E>();
  const long long R = varlen_rows(B, vl.total_q);
  const size_t rows = size_t(H) * size_t(R);
  float* dq_acc = static_cast<float*>(workspace);
  float* nlse2 = dq_acc + rows * D;
  float* ndelta = nlse2 + rows;
  {
    const size_t per_block = 8 * bwd::kPreRows;  // 8 warps of kPreRows rows (R is a multiple of 4)
    const unsigned blocks = unsigned((rows + per_block - 1) / per_block);
    bwd::attn_bwd_pre_varlen_kernel<D, E><<<blocks, 256, 0, stream>>>(
        static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), lse, nlse2, ndelta,
        dq_acc, vl.cu_q, vl.cu_k, B, H, vl.total_q, vl.total_k, vl.max_q, vl.max_k, int(R),
        st.err);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
  }
  alignas(64) CUtensorMap mq, mk, mv, mdo, mdq;
  if (make_map(&mq, q, 1, vl.total_q, H, D, dt) != ATTN_OK ||
      make_map(&mk, k, 1, vl.total_k, Hk, D, dt) != ATTN_OK ||
      make_map(&mv, v, 1, vl.total_k, Hk, D, dt) != ATTN_OK ||
      make_map(&mdo, dout, 1, vl.total_q, H, D, dt) != ATTN_OK ||
      make_dq_map(&mdq, dq_acc, (long long)rows, D) != ATTN_OK)
    return ATTN_ERR_LAUNCH;
  bwd::Params p;
  p.dk = static_cast<uint16_t*>(dk);
  p.dv = static_cast<uint16_t*>(dv);
  p.nlse2 = nlse2;
  p.ndelta = ndelta;
  p.dq_acc = dq_acc;
  p.B = B;
  p.H = H;
  p.Sq = vl.max_q;
  p.Sk = vl.max_k;
  p.Sq_pad = 0;
  p.cu_q = vl.cu_q;
  p.cu_k = vl.cu_k;
  p.total_q = vl.total_q;
  p.total_k = vl.total_k;
  p.R = int(R);
  p.Hk = Hk;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.win_left = win_left;
  p.win_right = win_right;
  p.err = st.err;
  p.timeout_ns = kTimeoutNs;
  // Up to kCompactMaxB sequences: one CTA per key tile that has work (at most
  // ceil(total_k / 128) + B of them); otherwise the longest sequence's tile
  // count for every sequence.
  p.compact = B <= kCompactMaxB ? 1 : 0;
  // chunked block order over the K/V heads (Q, dO and the dQ accumulator of the
  // query heads each serves, every sequence's rows)
  p.order_chunk = order_chunk(double(H / Hk) * double(vl.total_q) * D * (2.0 + 2.0 + 4.0),
                              p.compact ? Hk : Hk * B);
  dim3 grid = p.compact ? dim3((vl.total_k + bwd::BN - 1) / bwd::BN + B, Hk, 1)
                        : dim3((vl.max_k + bwd::BN - 1) / bwd::BN, Hk, B);
  bwd::attn_bwd_main_kernel<D, E, true>
      <<<grid, bwd::kThreads, bwd::Cfg<D>::kSmemBytes, stream>>>(mq, mk, mv, mdo, mdq, p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
  const long long total = (long long)vl.total_q * H * (D / 8);
  bwd::attn_bwd_dq_varlen_kernel<D, E><<<unsigned((total + 255) / 256), 256, 0, stream>>>(
      dq_acc, static_cast<uint16_t*>(dq), vl.cu_q, vl.cu_k, B, H, vl.total_q, vl.total_k,
      vl.max_q, vl.max_k, int(R), scale);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

// Decode: the key range of each (batch, K/V head) is cut into splits of whole
// 128-key tiles, one CTA each.  The split length minimises the estimated time
// ceil(CTAs / SMs) x (tiles per split + 3) (the + 3: a CTA's start-up and
// pipeline fill, measured at about three tiles' time), so the last wave of
// CTAs is not left mostly empty.  Splits
// have at least two tiles unless the cache has one; the workspace is sized for
// the largest split count this allows.
struct DecodePlan {
  int nsplit, tiles_per_split;
};
DecodePlan decode_plan(int B, int Smax, int Hk, int num_sms) {
  const int tiles = (Smax + dec::BN - 1) / dec::BN;
  const long long pairs = (long long)B * Hk;
  DecodePlan best{tiles, 1};
  long long best_cost = -1;
  for (int tps = tiles > 1 ? 2 : 1; tps <= tiles; ++tps) {
    const int nsplit = (tiles + tps - 1) / tps;
    const long long waves = (pairs * nsplit + num_sms - 1) / num_sms;
    const long long cost = waves * (tps + 3);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = {nsplit, tps};
    }
  }
  return best;
}
int decode_max_splits(int Smax) {
  const int tiles = (Smax + dec::BN - 1) / dec::BN;
  return tiles > 1 ? (tiles + 1) / 2 : 1;
}
size_t decode_workspace_bytes(int B, int Sq, int Smax, int H, int Hk, int D) {
  const size_t rows = size_t(B) * H * Sq * decode_max_splits(Smax);
  return ((rows * D * 4 + 255) / 256) * 256 + rows * 4;
}

template <int D, class E>
attn_status launch_decode(const DeviceState& st, const void* q, const void* kc, const void* vc,
                          const int* seqlens, void* o, float* lse, int B, int Sq, int Smax,
                          int H, int Hk, float scale, int causal, void* workspace,
                          cudaStream_t stream) {
  constexpr CUtensorMapDataType dt = tmap_type<E>();
  const int group = H / Hk;
  alignas(64) CUtensorMap mq, mk, mv;
  {
    // the K/V head's query heads at every new position: box (64 d, group heads, Sq rows)
    const cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(Sq), cuuint64_t(B)};
    const cuuint64_t strides[3] = {cuuint64_t(D) * 2, cuuint64_t(H) * D * 2,
                                   cuuint64_t(Sq) * H * D * 2};
    const cuuint32_t box[4] = {64, cuuint32_t(group), cuuint32_t(Sq), 1};
    if (encode_cached(&mq, dt, 4, q, dims, strides, box) != ATTN_OK) return ATTN_ERR_LAUNCH;
  }
  if (make_map(&mk, kc, B, Smax, Hk, D, dt) != ATTN_OK ||
      make_map(&mv, vc, B, Smax, Hk, D, dt) != ATTN_OK)
    return ATTN_ERR_LAUNCH;
  // keys on the tensor-memory lanes (at most 16 query rows per K/V head): at
  // head_dim 64 two CTAs share an SM, so a wave holds twice the SM count
  const bool keys_on_lanes = group * Sq <= dec::t16::kRows;
  const int sms = st.num_sms > 0 ? st.num_sms : 148;
  const DecodePlan plan =
      decode_plan(B, Smax, Hk, keys_on_lanes ? sms * dec::t16::Cfg<D>::kCtasPerSm : sms);
  // partial results are laid out for the largest split count (the workspace size)
  const size_t rows = size_t(B) * H * Sq * decode_max_splits(Smax);
  dec::Params p;
  p.seqlens = seqlens;
  p.opart = static_cast<float*>(workspace);
  p.lsepart = p.opart + ((rows * D * 4 + 255) / 256) * 256 / 4;
  p.B = B;
  p.Sq = Sq;
  p.Smax = Smax;
  p.H = H;
  p.Hk = Hk;
  p.group = group;
  p.nsplit = plan.nsplit;
  p.tiles_per_split = plan.tiles_per_split;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal ? 1 : 0;
  p.err = st.err;
  p.timeout_ns = kTimeoutNs;
  // at most 16 query rows per K/V head (one new token, up to 16 query heads
  // each): keys on the tensor-memory lanes; otherwise query rows on the lanes
  if (keys_on_lanes) {
    dec::t16::attn_decode_t16_kernel<D, E><<<dim3(plan.nsplit, Hk, B), dec::t16::kThreads,
                                               dec::t16::Cfg<D>::kSmemBytes, stream>>>(mq, mk, mv,
                                                                                       p);
  } else {
    dec::attn_decode_kernel<D, E><<<dim3(plan.nsplit, Hk, B), dec::kThreads,
                                    dec::Cfg<D>::kSmemBytes, stream>>>(mq, mk, mv, p);
  }
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
  // The combine is a programmatic dependent of the split kernel: its launch
  // overlaps the split kernel's tail, and it waits for that grid's results.
  const long long nrow = (long long)B * H * Sq;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned((nrow + 7) / 8));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e =
      cudaLaunchKernelEx(&cfg, dec::attn_decode_combine_kernel<D, E>,
                         static_cast<const float*>(p.opart), static_cast<const float*>(p.lsepart),
                         static_cast<uint16_t*>(o), lse, B, Sq, H, plan.nsplit);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? ATTN_OK : ATTN_ERR_LAUNCH;
}

attn_status check_workspace(const void* workspace, size_t bytes, int B, int Sq, int H, int D) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      bytes < workspace_bytes(B, Sq, H, D))
    return ATTN_ERR_WORKSPACE;
  return ATTN_OK;
}

bool all_on_device(std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs)
    if (!on_current_device(p)) return false;
  return true;
}

// ---------------------------------------------------------------------------
// Padded batches: the real rows gathered into packed tensors in the caller's
// workspace, the variable-length kernels run on those, the results scattered
// back with padding rows cleared.
// ---------------------------------------------------------------------------
constexpr int kPackTail = 128;  // cleared rows after the last packed row (a ragged tile's reach)

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace of a padded call: [cu_q][cu_k][packed tensors ...][varlen backward workspace].
struct PaddedLayout {
  size_t cu_q, cu_k, q, k, v, o, lse, dout, dq, dk, dv, bwd_ws, total;
};

PaddedLayout padded_layout(int B, int Sq, int Sk, int H, int Hk, int D, bool backward) {
  PaddedLayout L{};
  const size_t nq = size_t(B) * Sq * H * D * 2, nk = size_t(B) * Sk * Hk * D * 2;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  L.cu_q = take(size_t(B + 2) * 4);
  L.cu_k = take(size_t(B + 2) * 4);
  L.q = take(nq);
  L.k = take(nk);
  L.v = take(nk);
  L.o = take(nq);
  L.lse = take(size_t(H) * B * Sq * 4);
  if (backward) {
    L.dout = take(nq);
    L.dq = take(nq);
    L.dk = take(nk);
    L.dv = take(nk);
    L.bwd_ws = take(varlen_workspace_bytes(B, B * Sq, H, D));
  }
  L.total = off;
  return L;
}

attn_status check_padded(int B, int Sq, int Sk, int H, int Hk, int D, float scale, int win_left,
                         int win_right) {
  attn_status s = check_common(B, Sq, Sk, H, D, scale, win_left, win_right, Hk);
  if (s != ATTN_OK) return s;
  // the packed tensors and the varlen row layout must stay below 2^31 elements
  return check_varlen(B, B * Sq, B * Sk, Sq, Sk, H, Hk, D, scale, win_left, win_right);
}

template <int D>
attn_status launch_pack(const void* src, void* dst, const int* cu, int B, int S, int NH,
                        cudaStream_t cs) {
  const long long warps = (long long)B * S + kPackTail;
  padded::pack_rows_kernel<D><<<unsigned((warps + 7) / 8), 256, 0, cs>>>(
      static_cast<const uint16_t*>(src), static_cast<uint16_t*>(dst), cu, B, S, NH,
      (long long)B * S, kPackTail);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

template <int D>
attn_status launch_unpack(const void* src, void* dst, const int* cu, int B, int S, int NH,
                          cudaStream_t cs) {
  const long long warps = (long long)B * S;
  padded::unpack_rows_kernel<D><<<unsigned((warps + 7) / 8), 256, 0, cs>>>(
      static_cast<const uint16_t*>(src), static_cast<uint16_t*>(dst), cu, B, S, NH);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

attn_status launch_scans(const int* len_q, const int* len_k, int* cu_q, int* cu_k, int B, int Sq,
                         int Sk, uint32_t* err, cudaStream_t cs) {
  padded::seqlens_scan_kernel<<<1, 32, 0, cs>>>(len_q, B, Sq, cu_q, err);
  padded::seqlens_scan_kernel<<<1, 32, 0, cs>>>(len_k, B, Sk, cu_k, err);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

// ---------------------------------------------------------------------------
// Scratch for attn_bwd_noalloc: one statically declared device array per GPU.
// In host code `g_noalloc_scratch` is only a host-side stand-in for the
// symbol, never a device address; its device address is looked up once per
// device with cudaGetSymbolAddress (with that device current) and cached.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

struct ScratchState {
  bool init = false;
  void* ptr = nullptr;
};
ScratchState g_scratch[kMaxDevices];

attn_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  ScratchState& s = g_scratch[dev];
  if (!s.init) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return ATTN_ERR_LAUNCH;
    s.ptr = ptr;
    s.init = true;
  }
  *out = s.ptr;
  return ATTN_OK;
}

__global__ void attn_timeout_selftest_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  Bounded bw{&abort_flag, err, limit_ns};
  // Nothing ever arrives on `bar`, so this wait runs out after limit_ns.
  bw.wait(smem_u32(&bar), 0, 99);
}

}  // namespace

extern "C" {

const char* attn_status_string(attn_status s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_NULLPTR: return "a required pointer is NULL";
    case ATTN_ERR_SHAPE: return "bad shape or scale (B, H, Sq, Sk >= 1, sizes < 2^31, scale finite > 0)";
    case ATTN_ERR_HEADDIM:
      return "head_dim must be 64 or 128 (or 256 for the dense forward and backward)";
    case ATTN_ERR_ALIGN: return "tensor pointers must be 16-byte aligned";
    case ATTN_ERR_WINDOW: return "window sizes must be -1 (unbounded) or >= 0";
    case ATTN_ERR_ARCH: return "the current device is not compute capability 10.0 (sm_100a)";
    case ATTN_ERR_DEVICE: return "a pointer is not device memory of the current GPU";
    case ATTN_ERR_LAUNCH: return "a CUDA call failed (descriptor encoding or kernel launch)";
    case ATTN_ERR_TIMEOUT: return "a device-side bounded wait ran out";
    case ATTN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case ATTN_ERR_SCRATCH:
      return "backward scratch for this problem exceeds the 64 MiB built into attn_bwd_noalloc "
             "(call attn_bwd with a workspace instead)";
    case ATTN_ERR_DTYPE: return "dtype must be ATTN_DTYPE_BF16 (0) or ATTN_DTYPE_F16 (1)";
    case ATTN_ERR_SEQLENS:
      return "cu_seqlens found malformed on the device (not 0 <= cu[b] <= cu[b+1] <= total, or "
             "a sequence longer than its max_seqlen); the malformed sequences were skipped";
  }
  return "unknown status";
}

attn_status attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int Sq, int Sk, int H, int Hk, int D, int dtype, float scale, int causal,
                        int win_left, int win_right, void* stream) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_NULLPTR;
  attn_status s = check_common(B, Sq, Sk, H, D, scale, win_left, win_right, Hk, true);
  if (s != ATTN_OK) return s;
  if ((s = check_dtype(dtype)) != ATTN_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return ATTN_ERR_ALIGN;
  DeviceState* st = nullptr;
  s = device_state(&st);
  if (s != ATTN_OK) return s;
  if (!all_on_device({q, k, v, o, lse})) return ATTN_ERR_DEVICE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (D == 256) {
    return dtype == ATTN_DTYPE_F16
               ? launch_fwd_d256<ElemF16>(*st, q, k, v, o, lse, B, Sq, Sk, H, Hk, scale, causal,
                                          win_left, win_right, cs)
               : launch_fwd_d256<ElemBF16>(*st, q, k, v, o, lse, B, Sq, Sk, H, Hk, scale, causal,
                                           win_left, win_right, cs);
  }
  return dispatch(D, dtype, [&](auto d, auto e) {
    return launch_fwd<decltype(d)::value, decltype(e)>(*st, q, k, v, o, lse, B, Sq, Sk, H, Hk,
                                                       scale, causal, win_left, win_right, cs);
  });
}

attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int Sq, int Sk, int H, int D, float scale, int causal, int win_left,
                     int win_right, void* stream) {
  return attn_fwd_ex(q, k, v, o, lse, B, Sq, Sk, H, H, D, ATTN_DTYPE_BF16, scale, causal,
                     win_left, win_right, stream);
}

size_t attn_bwd_workspace_size(int B, int Sq, int H, int D) {
  if (B < 1 || Sq < 1 || H < 1 || (D != 64 && D != 128 && D != 256)) return 0;
  return workspace_bytes(B, Sq, H, D);
}

attn_status attn_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                        int Sq, int Sk, int H, int Hk, int D, int dtype, float scale, int causal,
                        int win_left, int win_right, void* workspace, size_t workspace_size,
                        void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return ATTN_ERR_NULLPTR;
  attn_status s = check_common(B, Sq, Sk, H, D, scale, win_left, win_right, Hk, true);
  if (s != ATTN_OK) return s;
  if ((s = check_dtype(dtype)) != ATTN_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return ATTN_ERR_ALIGN;
  s = check_workspace(workspace, workspace_size, B, Sq, H, D);
  if (s != ATTN_OK) return s;
  DeviceState* st = nullptr;
  s = device_state(&st);
  if (s != ATTN_OK) return s;
  if (!all_on_device({q, k, v, o, dout, lse, dq, dk, dv, workspace})) return ATTN_ERR_DEVICE;
  return run_backward(*st, q, k, v, o, dout, lse, dq, dk, dv, B, Sq, Sk, H, Hk, D, dtype, scale,
                      causal, win_left, win_right, carve(workspace, B, Sq, H, D),
                      static_cast<cudaStream_t>(stream));
}

attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, void* dq, void* dk, void* dv, int B, int Sq, int Sk, int H,
                     int D, float scale, int causal, int win_left, int win_right, void* workspace,
                     size_t workspace_size, void* stream) {
  return attn_bwd_ex(q, k, v, o, dout, lse, dq, dk, dv, B, Sq, Sk, H, H, D, ATTN_DTYPE_BF16,
                     scale, causal, win_left, win_right, workspace, workspace_size, stream);
}

attn_status attn_fwd_varlen(const void* q, const void* k, const void* v,
                            const int* cu_seqlens_q, const int* cu_seqlens_k, void* o, float* lse,
                            int B, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                            int H, int Hk, int D, int dtype, float scale, int causal,
                            int win_left, int win_right, void* stream) {
  if (!q || !k || !v || !cu_seqlens_q || !cu_seqlens_k || !o || !lse) return ATTN_ERR_NULLPTR;
  attn_status s = check_varlen(B, total_q, total_k, max_seqlen_q, max_seqlen_k, H, Hk, D, scale,
                               win_left, win_right);
  if (s != ATTN_OK) return s;
  if ((s = check_dtype(dtype)) != ATTN_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse) ||
      !aligned4(cu_seqlens_q) || !aligned4(cu_seqlens_k))
    return ATTN_ERR_ALIGN;
  DeviceState* st = nullptr;
  s = device_state(&st);
  if (s != ATTN_OK) return s;
  if (!all_on_device({q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k})) return ATTN_ERR_DEVICE;
  const Varlen vl{cu_seqlens_q, cu_seqlens_k, total_q, total_k, max_seqlen_q, max_seqlen_k};
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return dispatch(D, dtype, [&](auto d, auto e) {
    return launch_fwd_varlen<decltype(d)::value, decltype(e)>(*st, q, k, v, o, lse, vl, B, H, Hk,
                                                              scale, causal, win_left, win_right,
                                                              cs);
  });
}

size_t attn_bwd_varlen_workspace_size(int B, int total_q, int H, int D) {
  if (B < 1 || total_q < 1 || H < 1 || (D != 64 && D != 128)) return 0;
  return varlen_workspace_bytes(B, total_q, H, D);
}

attn_status attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                            const void* dout, const float* lse, const int* cu_seqlens_q,
                            const int* cu_seqlens_k, void* dq, void* dk, void* dv, int B,
                            int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int H,
                            int Hk, int D, int dtype, float scale, int causal, int win_left,
                            int win_right, void* workspace, size_t workspace_size,
                            void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !cu_seqlens_q || !cu_seqlens_k || !dq || !dk ||
      !dv)
    return ATTN_ERR_NULLPTR;
  attn_status s = check_varlen(B, total_q, total_k, max_seqlen_q, max_seqlen_k, H, Hk, D, scale,
                               win_left, win_right);
  if (s != ATTN_OK) return s;
  if ((s = check_dtype(dtype)) != ATTN_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned4(lse) ||
      !aligned4(cu_seqlens_q) || !aligned4(cu_seqlens_k))
    return ATTN_ERR_ALIGN;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_size < varlen_workspace_bytes(B, total_q, H, D))
    return ATTN_ERR_WORKSPACE;
  DeviceState* st = nullptr;
  s = device_state(&st);
  if (s != ATTN_OK) return s;
  if (!all_on_device({q, k, v, o, dout, lse, cu_seqlens_q, cu_seqlens_k, dq, dk, dv, workspace}))
    return ATTN_ERR_DEVICE;
  const Varlen vl{cu_seqlens_q, cu_seqlens_k, total_q, total_k, max_seqlen_q, max_seqlen_k};
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return dispatch(D, dtype, [&](auto d, auto e) {
    return run_backward_varlen<decltype(d)::value, decltype(e)>(
        *st, q, k, v, o, dout, lse, dq, dk, dv, vl, B, H, Hk, scale, causal, win_left, win_right,
        workspace, cs);
  });
}

attn_status attn_bwd_preprocess_ex(const void* o, const void* dout, const float* lse, int B,
                                   int Sq, int H, int D, int dtype, void* workspace,
                                   size_t workspace_size, void* stream) {
  if (!o || !dout || !lse) return ATTN_ERR_NULLPTR;
  attn_status s = check_common(B, Sq, 1, H, D, 1.0f, -1, -1, -1, true);
  if (s != ATTN_OK) return s;
  if ((s = check_dtype(dtype)) != ATTN_OK) return s;
  if (!aligned16(o) || !aligned16(dout) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return ATTN_ERR_ALIGN;
  s = check_workspace(workspace, workspace_size, B, Sq, H, D);
  if (s != ATTN_OK) return s;
  DeviceState* st = nullptr;
  s = device_state(&st);
  if (s != ATTN_OK) return s;
  if (!all_on_device({o, dout, lse, workspace})) return ATTN_ERR_DEVICE;
  const Workspace w = carve(workspace, B, Sq, H, D);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return dispatch_d256(D, dtype, [&](auto d, auto e) {
    return launch_bwd_pre<decltype(d)::value, decltype(e)>(o, dout, lse, B, Sq, H, w, cs);
  });
}

attn_status attn_bwd_preprocess(const void* o, const void* dout, const float* lse, int B, int Sq,
                                int H, int D, void* workspace, size_t workspace_size,
                                void* stream) {
  return attn_bwd_preprocess_ex(o, dout, lse, B, Sq, H, D, ATTN_DTYPE_BF16, workspace,
                                workspace_size, stream);
}

attn_status attn_bwd_main_ex(const void* q, const void* k, const void* v, const void* dout,
                             void* dk, void* dv, int B, int Sq, int Sk, int H, int Hk, int D,
                             int dtype, float scale, int causal, int win_left, int win_right,
                             void* workspace, size_t workspace_size, void* stream) {
  if (!q || !k || !v || !dout || !dk || !dv) return ATTN_ERR_NULLPTR;
  attn_status s = check_common(B, Sq, Sk, H, D, scale, win_left, win_right, Hk, true);
  if (s != ATTN_OK) return s;
  if ((s = check_dtype(dtype)) != ATTN_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dk) ||
      !aligned16(dv))
    return ATTN_ERR_ALIGN;
  s = check_workspace(workspace, workspace_size, B, Sq, H, D);
  if (s != ATTN_OK) return s;
  DeviceState* st = nullptr;
  s = device_state(&st);
  if (s != ATTN_OK) return s;
  if (!all_on_device({q, k, v, dout, dk, dv, workspace})) return ATTN_ERR_DEVICE;
  const Workspace w = carve(workspace, B, Sq, H, D);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return dispatch_d256(D, dtype, [&](auto d, auto e) {
    return launch_bwd_main_any<decltype(d)::value, decltype(e)>(*st, q, k, v, dout, dk, dv, B, Sq,
                                                            Sk, H, Hk, scale, causal, win_left,
                                                            win_right, w, cs);
  });
}

attn_status attn_bwd_main(const void* q, const void* k, const void* v, const void* dout,
                          void* dk, void* dv, int B, int Sq, int Sk, int H, int D, float scale,
                          int causal, int win_left, int win_right, void* workspace,
                          size_t workspace_size, void* stream) {
  return attn_bwd_main_ex(q, k, v, dout, dk, dv, B, Sq, Sk, H, H, D, ATTN_DTYPE_BF16, scale,
                          causal, win_left, win_right, workspace, workspace_size, stream);
}

attn_status attn_bwd_dq_finalize_ex(void* dq, int B, int Sq, int H, int D, int dtype,
                                    float scale, void* workspace, size_t workspace_size,
                                    void* stream) {
  if (!dq) return ATTN_ERR_NULLPTR;
  attn_status s = check_common(B, Sq, 1, H, D, scale, -1, -1, -1, true);
  if (s != ATTN_OK) return s;
  if ((s = check_dtype(dtype)) != ATTN_OK) return s;
  if (!aligned16(dq)) return ATTN_ERR_ALIGN;
  s = check_workspace(workspace, workspace_size, B, Sq, H, D);
  if (s != ATTN_OK) return s;
  DeviceState* st = nullptr;
  s = device_state(&st);
  if (s != ATTN_OK) return s;
  if (!all_on_device({dq, workspace})) return ATTN_ERR_DEVICE;
  const Workspace w = carve(workspace, B, Sq, H, D);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return dispatch_d256(D, dtype, [&](auto d, auto e) {
    return launch_bwd_dq<decltype(d)::value, decltype(e)>(dq, B, Sq, H, scale, w, cs);
  });
}

attn_status attn_bwd_dq_finalize(void* dq, int B, int Sq, int H, int D, float scale,
                                 void* workspace, size_t workspace_size, void* stream) {
  return attn_bwd_dq_finalize_ex(dq, B, Sq, H, D, ATTN_DTYPE_BF16, scale, workspace,
                                 workspace_size, stream);
}

attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                             const void* dout, const float* lse, void* dq, void* dk, void* dv,
                             int B, int Sq, int Sk, int H, int D, float scale, int causal,
                             int win_left, int win_right, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return ATTN_ERR_NULLPTR;
  attn_status s = check_common(B, Sq, Sk, H, D, scale, win_left, win_right, -1, true);
  if (s != ATTN_OK) return s;
  if (workspace_bytes(B, Sq, H, D) > ATTN_NOALLOC_SCRATCH_BYTES) return ATTN_ERR_SCRATCH;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return ATTN_ERR_ALIGN;
  DeviceState* st = nullptr;
  s = device_state(&st);
  if (s != ATTN_OK) return s;
  if (!all_on_device({q, k, v, o, dout, lse, dq, dk, dv})) return ATTN_ERR_DEVICE;
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != ATTN_OK) return s;
  // The preprocess kernel rewrites Delta and LSE rows and zeroes the dQ
  // accumulator, so nothing left in the scratch by an earlier call is read.
  return run_backward(*st, q, k, v, o, dout, lse, dq, dk, dv, B, Sq, Sk, H, H, D,
                      ATTN_DTYPE_BF16, scale, causal, win_left, win_right,
                      carve(scratch, B, Sq, H, D), static_cast<cudaStream_t>(stream));
}

size_t attn_decode_workspace_size(int B, int Sq, int Smax, int H, int Hk, int D) {
  if (B < 1 || Sq < 1 || Smax < 1 || H < 1 || Hk < 1 || H % Hk || (D != 64 && D != 128))
    return 0;
  return decode_workspace_bytes(B, Sq, Smax, H, Hk, D);
}

attn_status attn_decode(const void* q, const void* k_cache, const void* v_cache,
                        const int* cache_seqlens, void* o, float* lse, int B, int Sq, int Smax,
                        int H, int Hk, int D, int dtype, float scale, int causal,
                        void* workspace, size_t workspace_size, void* stream) {
  if (!q || !k_cache || !v_cache || !cache_seqlens || !o || !lse) return ATTN_ERR_NULLPTR;
  attn_status s = check_common(B, Sq, Smax, H, D, scale, -1, -1, Hk);
  if (s != ATTN_OK) return s;
  if ((H / Hk) * Sq > dec::BM) return ATTN_ERR_SHAPE;  // the group's rows fill one 128-row tile
  if ((s = check_dtype(dtype)) != ATTN_OK) return s;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u))
    return ATTN_ERR_ALIGN;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_size < decode_workspace_bytes(B, Sq, Smax, H, Hk, D))
    return ATTN_ERR_WORKSPACE;
  DeviceState* st = nullptr;
  s = device_state(&st);
  if (s != ATTN_OK) return s;
  if (!all_on_device({q, k_cache, v_cache, cache_seqlens, o, lse, workspace}))
    return ATTN_ERR_DEVICE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return dispatch(D, dtype, [&](auto d, auto e) {
    return launch_decode<decltype(d)::value, decltype(e)>(*st, q, k_cache, v_cache,
                                                          cache_seqlens, o, lse, B, Sq, Smax, H,
                                                          Hk, scale, causal, workspace, cs);
  });
}

attn_status attn_decode_split_plan(int B, int Smax, int Hk, int num_sms, int* nsplit,
                                   int* tiles_per_split) {
  if (!nsplit || !tiles_per_split) return ATTN_ERR_NULLPTR;
  if (B < 1 || Smax < 1 || Hk < 1 || num_sms < 1) return ATTN_ERR_SHAPE;
  const DecodePlan plan = decode_plan(B, Smax, Hk, num_sms);
  *nsplit = plan.nsplit;
  *tiles_per_split = plan.tiles_per_split;
  return ATTN_OK;
}

size_t attn_fwd_padded_workspace_size(int B, int Sq, int Sk, int H, int Hk, int D) {
  if (check_padded(B, Sq, Sk, H, Hk, D, 1.0f, -1, -1) != ATTN_OK) return 0;
  return padded_layout(B, Sq, Sk, H, Hk, D, false).total;
}

size_t attn_bwd_padded_workspace_size(int B, int Sq, int Sk, int H, int Hk, int D) {
  if (check_padded(B, Sq, Sk, H, Hk, D, 1.0f, -1, -1) != ATTN_OK) return 0;
  return padded_layout(B, Sq, Sk, H, Hk, D, true).total;
}

attn_status attn_fwd_padded(const void* q, const void* k, const void* v, const int* seqlens_q,
                            const int* seqlens_k, void* o, float* lse, int B, int Sq, int Sk,
                            int H, int Hk, int D, int dtype, float scale, int causal,
                            int win_left, int win_right, void* workspace, size_t workspace_size,
                            void* stream) {
  if (!q || !k || !v || !seqlens_q || !seqlens_k || !o || !lse) return ATTN_ERR_NULLPTR;
  attn_status s = check_padded(B, Sq, Sk, H, Hk, D, scale, win_left, win_right);
  if (s != ATTN_OK) return s;
  if ((s = check_dtype(dtype)) != ATTN_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse) ||
      !aligned4(seqlens_q) || !aligned4(seqlens_k))
    return ATTN_ERR_ALIGN;
  const PaddedLayout L = padded_layout(B, Sq, Sk, H, Hk, D, false);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_size < L.total)
    return ATTN_ERR_WORKSPACE;
  DeviceState* st = nullptr;
  s = device_state(&st);
  if (s != ATTN_OK) return s;
  if (!all_on_device({q, k, v, o, lse, seqlens_q, seqlens_k, workspace})) return ATTN_ERR_DEVICE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* cu_q = reinterpret_cast<int*>(ws + L.cu_q);
  int* cu_k = reinterpret_cast<int*>(ws + L.cu_k);
  const Varlen vl{cu_q, cu_k, B * Sq, B * Sk, Sq, Sk};
  if ((s = launch_scans(seqlens_q, seqlens_k, cu_q, cu_k, B, Sq, Sk, st->err, cs)) != ATTN_OK)
    return s;
  return dispatch(D, dtype, [&](auto d, auto e) {
    constexpr int DD = decltype(d)::value;
    using E = decltype(e);
    attn_status r = launch_pack<DD>(q, ws + L.q, cu_q, B, Sq, H, cs);
    if (r == ATTN_OK) r = launch_pack<DD>(k, ws + L.k, cu_k, B, Sk, Hk, cs);
    if (r == ATTN_OK) r = launch_pack<DD>(v, ws + L.v, cu_k, B, Sk, Hk, cs);
    if (r == ATTN_OK)
      r = launch_fwd_varlen<DD, E>(*st, ws + L.q, ws + L.k, ws + L.v, ws + L.o,
                                   reinterpret_cast<float*>(ws + L.lse), vl, B, H, Hk, scale,
                                   causal, win_left, win_right, cs);
    if (r == ATTN_OK) r = launch_unpack<DD>(ws + L.o, o, cu_q, B, Sq, H, cs);
    if (r == ATTN_OK) {
      const long long n = (long long)B * H * Sq;
      padded::unpack_lse_kernel<<<unsigned((n + 255) / 256), 256, 0, cs>>>(
          reinterpret_cast<const float*>(ws + L.lse), lse, cu_q, B, Sq, H, (long long)B * Sq);
      if (cudaGetLastError() != cudaSuccess) r = ATTN_ERR_LAUNCH;
    }
    return r;
  });
}

attn_status attn_bwd_padded(const void* q, const void* k, const void* v, const void* o,
                            const void* dout, const float* lse, const int* seqlens_q,
                            const int* seqlens_k, void* dq, void* dk, void* dv, int B, int Sq,
                            int Sk, int H, int Hk, int D, int dtype, float scale, int causal,
                            int win_left, int win_right, void* workspace, size_t workspace_size,
                            void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !seqlens_q || !seqlens_k || !dq || !dk || !dv)
    return ATTN_ERR_NULLPTR;
  attn_status s = check_padded(B, Sq, Sk, H, Hk, D, scale, win_left, win_right);
  if (s != ATTN_OK) return s;
  if ((s = check_dtype(dtype)) != ATTN_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned4(lse) ||
      !aligned4(seqlens_q) || !aligned4(seqlens_k))
    return ATTN_ERR_ALIGN;
  const PaddedLayout L = padded_layout(B, Sq, Sk, H, Hk, D, true);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_size < L.total)
    return ATTN_ERR_WORKSPACE;
  DeviceState* st = nullptr;
  s = device_state(&st);
  if (s != ATTN_OK) return s;
  if (!all_on_device({q, k, v, o, dout, lse, seqlens_q, seqlens_k, dq, dk, dv, workspace}))
    return ATTN_ERR_DEVICE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* cu_q = reinterpret_cast<int*>(ws + L.cu_q);
  int* cu_k = reinterpret_cast<int*>(ws + L.cu_k);
  const Varlen vl{cu_q, cu_k, B * Sq, B * Sk, Sq, Sk};
  if ((s = launch_scans(seqlens_q, seqlens_k, cu_q, cu_k, B, Sq, Sk, st->err, cs)) != ATTN_OK)
    return s;
  float* lse_p = reinterpret_cast<float*>(ws + L.lse);
  return dispatch(D, dtype, [&](auto d, auto e) {
    constexpr int DD = decltype(d)::value;
    using E = decltype(e);
    attn_status r = launch_pack<DD>(q, ws + L.q, cu_q, B, Sq, H, cs);
    if (r == ATTN_OK) r = launch_pack<DD>(k, ws + L.k, cu_k, B, Sk, Hk, cs);
    if (r == ATTN_OK) r = launch_pack<DD>(v, ws + L.v, cu_k, B, Sk, Hk, cs);
    if (r == ATTN_OK) r = launch_pack<DD>(o, ws + L.o, cu_q, B, Sq, H, cs);
    if (r == ATTN_OK) r = launch_pack<DD>(dout, ws + L.dout, cu_q, B, Sq, H, cs);
    if (r == ATTN_OK) {
      const long long n = (long long)B * H * Sq;
      padded::pack_lse_kernel<<<unsigned((n + 255) / 256), 256, 0, cs>>>(
          lse, lse_p, cu_q, B, Sq, H, (long long)B * Sq);
      if (cudaGetLastError() != cudaSuccess) r = ATTN_ERR_LAUNCH;
    }
    if (r == ATTN_OK)
      r = run_backward_varlen<DD, E>(*st, ws + L.q, ws + L.k, ws + L.v, ws + L.o, ws + L.dout,
                                     lse_p, ws + L.dq, ws + L.dk, ws + L.dv, vl, B, H, Hk, scale,
                                     causal, win_left, win_right, ws + L.bwd_ws, cs);
    if (r == ATTN_OK) r = launch_unpack<DD>(ws + L.dq, dq, cu_q, B, Sq, H, cs);
    if (r == ATTN_OK) r = launch_unpack<DD>(ws + L.dk, dk, cu_k, B, Sk, Hk, cs);
    if (r == ATTN_OK) r = launch_unpack<DD>(ws + L.dv, dv, cu_k, B, Sk, Hk, cs);
    return r;
  });
}

attn_status attn_get_last_device_error(void) {
  DeviceState* st = nullptr;
  attn_status s = device_state(&st);
  if (s != ATTN_OK) return s;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_LAUNCH;
  uint32_t word = 0;
  if (cudaMemcpyFromSymbol(&word, g_attn_err, sizeof(word)) != cudaSuccess) return ATTN_ERR_LAUNCH;
  if (word == 0) return ATTN_OK;
  const uint32_t zero = 0;
  cudaMemcpyToSymbol(g_attn_err, &zero, sizeof(zero));
  if ((word & 0xFFu) == kErrTimeout) return ATTN_ERR_TIMEOUT;
  if ((word & 0xFFu) == kErrSeqlens) return ATTN_ERR_SEQLENS;
  return ATTN_ERR_LAUNCH;
}

attn_status attn_device_timeout_selftest(int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return ATTN_ERR_SHAPE;
  DeviceState* st = nullptr;
  attn_status s = device_state(&st);
  if (s != ATTN_OK) return s;
  attn_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      st->err, uint64_t(limit_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

}  // extern "C"
