// Host side of libmonoffn: the C ABI declared in include/mono_ffn.h — plan
// validation and allocation, the one-time weight repack, the per-step
// launches and the device error word.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "mono_ffn.h"
#include "cc_kernel.cuh"
#include "tc_kernel.cuh"
#include "tq_kernel.cuh"

using namespace mono;

namespace {

thread_local std::string g_plan_error;

struct LayerSlot {
  float* mix_w = nullptr;
  void* norm_w = nullptr;
  float* router_t = nullptr;
  float* bias = nullptr;
  uint8_t* gu = nullptr;
  uint8_t* dn = nullptr;
  float* gsc = nullptr;   // quantised tensor-core path: packed block scales (FP8 fp32, MXFP4 e8m0 chunks)
  float* dsc = nullptr;
  CUtensorMap tm_gu{}, tm_dn{};   // MXFP4: tensor maps of the packed codes
  bool packed = false;
  Taps taps{};
};

}  // namespace

struct mono_ffn_plan_s {
  mono_ffn_config cfg{};
  int wt = 0;
  bool tc = false;   // bf16 experts run on the tensor-core kernel
  bool tq = false;   // FP8 / MXFP4 experts run on the quantised tensor-core kernel
  int G = 0, nst = 0, slot_bytes = 0, regA_bytes = 0, ymax = 0, mix_ctas = 0, smem = 0;
  int gu_kc = 0, gu_nk = 0, gu_rc = 0, dn_kc = 0, dn_nk = 0, dn_rc = 0;
  long long gu_estride = 0, dn_estride = 0;
  std::vector<LayerSlot> layers;
  float* mix_part = nullptr;
  float* mix_tot = nullptr;
  void* abuf = nullptr;
  float* sq_part = nullptr;
  float* logits = nullptr;
  float* act = nullptr;
  float* yp = nullptr;
  uint8_t* actb = nullptr;
  float* gpart = nullptr;
  float* dpart = nullptr;
  uint32_t* gcnt = nullptr;
  uint32_t* xready = nullptr;
  uint32_t* dcnt = nullptr;
  size_t gcnt_n = 0, dcnt_n = 0;
  std::vector<float*> pend;
  void* xbuf[2] = {nullptr, nullptr};
  SyncBlock* sync = nullptr;
  ErrBlock* err = nullptr;
  void* stage_in = nullptr;
  void* stage_out = nullptr;
  int64_t packed_bytes = 0, scratch_bytes = 0;
  bool pdl_ok = true;   // a chain's later layers launch as programmatic dependents
  int fault_cta = -1;
  int fault_stage = 0;
  unsigned jitter_ns = 0;
  unsigned long long* trace = nullptr;
  std::string last_error;
};

namespace {

int elem_bits(int dt) { return dt == MONO_F32 ? 32 : dt == MONO_BF16 ? 16 : dt == MONO_FP8E4M3_B128 ? 8 : 4; }
int block_of(int dt) { return dt == MONO_FP8E4M3_B128 ? 128 : dt == MONO_MXFP4 ? 32 : 0; }
int unit_elems(int dt) { return 128 / elem_bits(dt); }   // elements per 16 bytes

// largest chunk <= target that divides K and keeps whole 16-byte units and scale blocks
int pick_kc(int dt, int K, int target) {
  int step = std::max(unit_elems(dt), block_of(dt));
  for (int kc = std::min(target, K) / step * step; kc >= step; kc -= step)
    if (K % kc == 0) return kc;
  return 0;
}

int code_bytes(int dt, int kc) { return (int)((long long)kc * elem_bits(dt) / 8); }
int scale_bytes(int dt, int kc) {
  if (dt == MONO_FP8E4M3_B128) return kc / 128 * 4;
  if (dt == MONO_MXFP4) return kc / 32;
  return 0;
}
int chunk_bytes(int dt, int kc) { return (int)align_up((size_t)code_bytes(dt, kc) + scale_bytes(dt, kc), 16); }

int fail(mono_ffn_plan_t* p, int code, const std::string& msg) {
  if (p) p->last_error = msg;
  else g_plan_error = msg;
  return code;
}

int cuda_fail(mono_ffn_plan_t* p, cudaError_t e, const char* what) {
  return fail(p, MONO_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

template <int WT>
void* kernel_ptr() {
  return reinterpret_cast<void*>(&mono_ffn_cc_kernel<WT>);
}

void* kernel_for(int wt, bool tc, bool tq) {
  if (tc) return reinterpret_cast<void*>(&mono_ffn_tc_kernel<W_BF16>);
  if (tq) return wt == W_FP8 ? reinterpret_cast<void*>(&mono_ffn_tq_kernel<W_FP8>)
                             : reinterpret_cast<void*>(&mono_ffn_tq_kernel<W_FP4>);
  switch (wt) {
    case W_F32: return kernel_ptr<W_F32>();
    case W_BF16: return kernel_ptr<W_BF16>();
    case W_FP8: return kernel_ptr<W_FP8>();
    default: return kernel_ptr<W_FP4>();
  }
}

// Tensor-core layout of one [E+1][rows][cols] bf16 matrix set: blocks of 128
// rows; inside a block, per contraction group kg (8 elements), the 16
// rowgroups of 8 rows as core matrices of 8 rows x 16 bytes, each rg taking
// rgb bytes (gate and up share one: sub = 0 or 128).  The 16-byte chunk of
// (e, row, kg) lands at
//   dst[((e * rows/128 + row/128) * cols/8 + kg) * 16 * rgb + ((row % 128) / 8) * rgb + sub + (row % 8) * 16].
__global__ void pack_tc_kernel(const uint16_t* src, uint8_t* dst, long long e1, int rows, int cols, int rgb, int sub) {
  const long long KG = cols / 8, NB = rows / 128;
  const long long n = e1 * rows * KG;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const long long kg = i % KG, row = (i / KG) % rows, e = i / (KG * rows);
    const uint4 v = *reinterpret_cast<const uint4*>(src + ((e * rows + row) * cols + kg * 8));
    const long long off = ((e * NB + row / 128) * KG + kg) * 16 * rgb + ((row % 128) / 8) * rgb + sub + (row % 8) * 16;
    *reinterpret_cast<uint4*>(dst + off) = v;
  }
}

// Quantised tensor-core layout of one [E+1][rows][row_bytes] code matrix set:
// units of 128 rows x ub bytes (128 contraction elements), the 16-byte chunk
// j of unit-row i at j * 2048 + i * 16 inside the unit's matrix slot msub:
//   dst[((e * rows/128 + row/128) * nu + u) * ustride + msub + j * 2048 + (row % 128) * 16]
__global__ void pack_tq_codes_kernel(const uint8_t* src, uint8_t* dst, long long e1, int rows, int row_bytes, int ub,
                                     long long ustride, int msub) {
  const int nch = row_bytes / 16, nu = row_bytes / ub, cpu = ub / 16, NB = rows / 128;
  const long long n = e1 * rows * nch;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int ch = (int)(i % nch);
    const long long row = (i / nch) % rows, e = i / ((long long)nch * rows);
    const int u = ch / cpu, j = ch % cpu;
    const uint4 v = *reinterpret_cast<const uint4*>(src + (e * rows + row) * row_bytes + (long long)ch * 16);
    const long long off = ((e * NB + row / 128) * nu + u) * ustride + msub + (long long)j * 2048 + (row % 128) * 16;
    *reinterpret_cast<uint4*>(dst + off) = v;
  }
}

// FP8 fp32 block scales [E+1][rows][cols/128] -> [E+1][rows/128][cols/128][nm * 128]
// (slot m = gate 0 / up 1 of a gate/up pair, or the single down matrix)
__global__ void pack_tq_scales_kernel(const float* src, float* dst, long long e1, int rows, int nu, int nm, int m) {
  const int NB = rows / 128;
  const long long n = e1 * rows * nu;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int u = (int)(i % nu);
    const long long row = (i / nu) % rows, e = i / ((long long)nu * rows);
    dst[((e * NB + row / 128) * nu + u) * (nm * 128) + m * 128 + row % 128] = src[(e * rows + row) * nu + u];
  }
}

// MXFP4 on the block-scaled tensor-core path, codes: one [E+1][rows][K/2]
// byte matrix set -> unit-matrices of 128 rows x 128 contraction elements,
// each 128 rows x 64 bytes row-major (the e2m1 stream as given, two codes a
// byte), unit-matrix (e, row block, unit u, slot msub of nm) at
//   dst[(((e * rows/128 + row/128) * nu + u) * nm + msub) * 8192 + (row % 128) * 64]
// so a 2-D tensor map of 64-byte rows reads a unit-matrix as one box.
__global__ void pack_mx_codes_kernel(const uint8_t* src, uint8_t* dst, long long e1, int rows, int row_bytes, int nm,
                                     int msub) {
  const int nu = row_bytes / 64, NB = rows / 128;
  const long long n = e1 * rows * nu * 4;   // 16-byte chunks
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int q = (int)(i & 3), u = (int)((i >> 2) % nu);
    const long long row = (i >> 2) / nu % rows, e = (i >> 2) / nu / rows;
    const uint4 v = *reinterpret_cast<const uint4*>(src + (e * rows + row) * row_bytes + (long long)u * 64 + q * 16);
    const long long um = ((e * NB + row / 128) * nu + u) * nm + msub;
    *reinterpret_cast<uint4*>(dst + um * 8192 + (row % 128) * 64 + q * 16) = v;
  }
}

// MXFP4 e8m0 block scales [E+1][rows][K/32] -> one 512-byte chunk per
// unit-matrix (same indexing as the codes), byte 16 a + 4 b + j = the scale
// of row 32 b + a of the block for K-block j of the unit: the layout that
// tcgen05.cp (32x128b, copied to all four lane quarters) turns into tensor-
// memory column b, lane a, byte j, which is where the block-scaled MMA reads
// row 32 b + a's scale for its K-step j.
__global__ void pack_mx_scales_kernel(const uint8_t* src, uint8_t* dst, long long e1, int rows, int ns, int nm,
                                      int msub) {
  const int nu = ns / 4, NB = rows / 128;
  const long long n = e1 * rows * ns;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int k = (int)(i % ns);
    const long long row = (i / ns) % rows, e = i / ns / rows;
    const int u = k / 4, j = k % 4, r = (int)(row % 128), a = r % 32, b = r / 32;
    const long long um = ((e * NB + row / 128) * nu + u) * nm + msub;
    dst[um * 512 + 16 * a + 4 * b + j] = src[(e * rows + row) * ns + k];
  }
}

// smallest and largest byte of n (for the MXFP4 scale range check)
__global__ void byte_range_kernel(const uint8_t* src, long long n, unsigned int* mm) {
  unsigned int lo = 255, hi = 0;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const unsigned int v = src[i];
    lo = min(lo, v);
    hi = max(hi, v);
  }
  atomicMin(&mm[0], lo);
  atomicMax(&mm[1], hi);
}

// ------------------------------------------------------------ pack kernels --

// Cut every [rows][in] matrix row into nk chunks of kc elements, each chunk
// followed by its block scales and padded to rc bytes; chunk (row, k) lands at
// dst + (row * nk + k) * item + sub.
__global__ void pack_rows_kernel(const uint8_t* codes, const uint8_t* scales, uint8_t* dst, long long rows,
                                 int nk, int cb, int sb, int rc, int item, int sub, int vec) {
  const long long nitems = rows * nk;
  const int lane = threadIdx.x & 31;
  long long w = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (; w < nitems; w += nw) {
    const long long row = w / nk;
    const int k = (int)(w % nk);
    const uint8_t* src = codes + row * (long long)cb * nk + (long long)k * cb;
    uint8_t* d = dst + (row * nk + k) * (long long)item + sub;
    if (vec) {
      for (int i = lane; i < cb / 16; i += 32)
        reinterpret_cast<uint4*>(d)[i] = reinterpret_cast<const uint4*>(src)[i];
    } else {
      for (int i = lane; i < cb; i += 32) d[i] = src[i];
    }
    if (sb) {
      const uint8_t* ss = scales + row * (long long)sb * nk + (long long)k * sb;
      for (int i = lane; i < sb; i += 32) d[cb + i] = ss[i];
    }
    for (int i = cb + sb + lane; i < rc; i += 32) d[i] = 0;
  }
}

__global__ void transpose_f32_kernel(const float* src, float* dst, int rows, int cols) {
  __shared__ float tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    int r = r0 + i, cc = c0 + threadIdx.x;
    if (r < rows && cc < cols) tile[i][threadIdx.x] = src[(size_t)r * cols + cc];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    int cc = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && cc < cols) dst[(size_t)cc * rows + r] = tile[threadIdx.x][i];
  }
}

int pack_matrix(mono_ffn_plan_t* p, const void* codes, const void* scales, uint8_t* dst, long long rows, int in,
                int kc, int nk, int rc, int item, int sub, cudaStream_t st) {
  const int dt = p->cfg.expert_dtype;
  const int cb = code_bytes(dt, kc), sb = scale_bytes(dt, kc);
  if (sb && !scales) return fail(p, MONO_ERR_INVALID_ARG, "pack: block scales are required for this expert format");
  (void)in;
  const int vec = ((uintptr_t)codes % 16 == 0) && (cb % 16 == 0);
  long long warps = rows * nk;
  long long blocks = std::min<long long>((warps + 7) / 8, 148LL * 32);
  pack_rows_kernel<<<(unsigned)blocks, 256, 0, st>>>((const uint8_t*)codes, (const uint8_t*)scales, dst, rows, nk, cb,
                                                     sb, rc, item, sub, vec);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? 0 : cuda_fail(p, e, "pack kernel launch");
}

// 2-D tensor map of packed MXFP4 unit-matrices: rows of 128 e2m1 codes (64
// bytes), `rows` of them; one box is a unit-matrix (128 rows).  Data type
// 16U4_ALIGN16B: in shared memory every 16 codes take a 16-byte slot (8 bytes
// of codes, then 8 unused), which is how the block-scaled MMA reads e2m1;
// with the 128-byte swizzle, so that a box is the MMA's swizzled K-major
// operand.
int make_f4_map(mono_ffn_plan_t* p, CUtensorMap* map, void* base, unsigned long long rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if (!enc) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
      return fail(p, MONO_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint64_t dims[2] = {128, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {64};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t es[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, base, dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(p, MONO_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return 0;
}

template <typename T>
int dalloc(mono_ffn_plan_t* p, T** ptr, size_t bytes, int64_t* acct) {
  if (bytes == 0) bytes = 16;
  cudaError_t e = cudaMalloc((void**)ptr, bytes);
  if (e != cudaSuccess) return fail(p, MONO_ERR_OOM, std::string("cudaMalloc of ") + std::to_string(bytes) + " bytes: " +
                                                         cudaGetErrorString(e));
  *acct += (int64_t)bytes;
  return 0;
}

}  // namespace

// ================================================================ the C ABI

extern "C" int mono_ffn_abi_version(void) { return 2; }

extern "C" const char* mono_ffn_last_error(const mono_ffn_plan_t* plan) {
  return plan ? plan->last_error.c_str() : g_plan_error.c_str();
}

extern "C" void mono_ffn_destroy(mono_ffn_plan_t* p) {
  if (!p) return;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(p->cfg.device);
  for (auto& l : p->layers) {
    cudaFree(l.mix_w);
    cudaFree(l.norm_w);
    cudaFree(l.router_t);
    cudaFree(l.bias);
    cudaFree(l.gu);
    cudaFree(l.dn);
    cudaFree(l.gsc);
    cudaFree(l.dsc);
  }
  for (float* q : p->pend) cudaFree(q);
  cudaFree(p->mix_part);
  cudaFree(p->mix_tot);
  cudaFree(p->abuf);
  cudaFree(p->sq_part);
  cudaFree(p->logits);
  cudaFree(p->act);
  cudaFree(p->yp);
  cudaFree(p->actb);
  cudaFree(p->gpart);
  cudaFree(p->dpart);
  cudaFree(p->gcnt);
  cudaFree(p->xready);
  cudaFree(p->dcnt);
  cudaFree(p->xbuf[0]);
  cudaFree(p->xbuf[1]);
  cudaFree(p->sync);
  cudaFree(p->err);
  cudaFree(p->stage_in);
  cudaFree(p->stage_out);
  cudaSetDevice(prev);
  delete p;
}

extern "C" int mono_ffn_plan(const mono_ffn_config* cfg_in, mono_ffn_plan_t** out) {
  g_plan_error.clear();
  if (!cfg_in || !out) return fail(nullptr, MONO_ERR_INVALID_ARG, "plan: NULL argument");
  *out = nullptr;
  mono_ffn_config cfg = *cfg_in;
  if (cfg.wait_timeout_us == 0) cfg.wait_timeout_us = 250000;
  std::string why;
  auto need = [&](bool ok, const std::string& m) {
    if (!ok) why += m + "\n";
  };
  const int dt = cfg.expert_dtype;
  need(cfg.hc == kS, "hc must be 4");
  need(cfg.hidden > 0 && cfg.inter > 0, "hidden and inter must be positive");
  need(cfg.n_routed >= 1 && cfg.n_routed <= kMaxE, "n_routed must be in [1, 1024]");
  need(cfg.top_k >= 1 && cfg.top_k <= std::min(cfg.n_routed, kMaxK), "top_k must be in [1, min(n_routed, 16)]");
  need(cfg.max_rows >= 1 && cfg.max_rows <= kMaxR, "max_rows must be in [1, 8]");
  need(cfg.n_layers >= 1, "n_layers must be >= 1");
  need(cfg.hc_dtype == MONO_F32 || cfg.hc_dtype == MONO_BF16, "hc_dtype must be F32 or BF16");
  need(cfg.norm_dtype == MONO_F32 || cfg.norm_dtype == MONO_BF16, "norm_dtype must be F32 or BF16");
  need(dt >= MONO_F32 && dt <= MONO_MXFP4, "expert_dtype unknown");
  need(!(cfg.hc_dtype == MONO_BF16 && !cfg.round_bf16), "bf16 residual streams need round_bf16 = 1");
  need(cfg.sinkhorn_iters >= 0, "sinkhorn_iters must be >= 0");
  need(cfg.dense == 0 || cfg.dense == 1, "dense must be 0 or 1");
  need(!cfg.dense || cfg.top_k == cfg.n_routed, "a dense layer takes every slot: top_k must equal n_routed");
  need(cfg.act_mx8 == 0 || cfg.act_mx8 == 1, "act_mx8 must be 0 or 1");
  need(!cfg.act_mx8 || (dt == MONO_MXFP4 && cfg.round_bf16 && cfg.hidden % 128 == 0 && cfg.inter % 128 == 0 &&
                        cfg.hidden <= kMx8MaxK && cfg.inter <= kMx8MaxK),
       "act_mx8 needs MXFP4 experts on the tensor cores (round_bf16, hidden and inter multiples of 128, at most " +
           std::to_string(kMx8MaxK) + ")");
  if (dt >= MONO_F32 && dt <= MONO_MXFP4 && cfg.hidden > 0 && cfg.inter > 0) {
    const int m = std::max(unit_elems(dt), block_of(dt));
    need(cfg.hidden % m == 0, "hidden must be a multiple of " + std::to_string(m) + " for this expert format");
    need(cfg.inter % m == 0, "inter must be a multiple of " + std::to_string(m) + " for this expert format");
    need(cfg.hidden % 8 == 0 && cfg.inter % 8 == 0, "hidden and inter must be multiples of 8");
    // MXFP4 on the tensor cores keeps one B-scale column per 128 of inter
    need(!(dt == MONO_MXFP4 && cfg.round_bf16 && cfg.hidden % 128 == 0 && cfg.inter % 128 == 0) ||
             cfg.inter <= kF4MaxI,
         "MXFP4 on the tensor cores takes inter <= " + std::to_string(kF4MaxI));
  }
  // the kernels partition every work list in 32-bit arithmetic: units x grid < 2^31
  need((long long)(cfg.max_rows * cfg.top_k + 1) * ((cfg.inter + 127) / 128) * ((cfg.hidden + 127) / 128) * 1024 <
           (1ll << 31),
       "hidden x inter too large for the work partition");
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) why += "no CUDA device\n";
  else if (cfg.device < 0 || cfg.device >= ndev) why += "device ordinal out of range\n";
  if (!why.empty()) return fail(nullptr, MONO_ERR_INVALID_ARG, why);

  cudaDeviceProp prop{};
  cudaGetDeviceProperties(&prop, cfg.device);
  if (prop.major != 10 || prop.minor != 0)
    return fail(nullptr, MONO_ERR_UNSUPPORTED_ARCH,
                "device " + std::to_string(cfg.device) + " is sm_" + std::to_string(prop.major) +
                    std::to_string(prop.minor) + "; this library is built for sm_100a only");
  if (!prop.cooperativeLaunch) return fail(nullptr, MONO_ERR_NOT_CORESIDENT, "device lacks cooperative launch");

  mono_ffn_plan_t* p = new mono_ffn_plan_s();
  p->cfg = cfg;
  p->wt = dt;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(cfg.device);
  const int H = cfg.hidden, I = cfg.inter, E = cfg.n_routed, K = cfg.top_k, RM = cfg.max_rows;

  // bf16 experts run on the tensor cores when the shapes allow it
  // whole 128-row blocks and 128-wide K units; n is the bf16 B operand
  p->tc = dt == MONO_BF16 && cfg.round_bf16 && H % 128 == 0 && I % 128 == 0;
  // FP8 / MXFP4 experts: converted to fp16 on the way into the tensor cores
  p->tq = (dt == MONO_FP8E4M3_B128 || dt == MONO_MXFP4) && cfg.round_bf16 && H % 128 == 0 && I % 128 == 0;
  const long long tq_mat = dt == MONO_FP8E4M3_B128 ? 16384 : 8192;   // one 128 x 128 unit of one matrix in HBM
  // chunking of the packed rows
  const int gu_target = dt == MONO_F32 ? 256 : dt == MONO_BF16 ? 512 : 1024;
  const int dn_target = dt == MONO_F32 ? 512 : dt == MONO_BF16 ? 1024 : 2048;
  p->gu_kc = pick_kc(dt, H, gu_target);
  p->dn_kc = pick_kc(dt, I, dn_target);
  p->gu_nk = H / p->gu_kc;
  p->dn_nk = I / p->dn_kc;
  p->gu_rc = chunk_bytes(dt, p->gu_kc);
  p->dn_rc = chunk_bytes(dt, p->dn_kc);
  p->gu_estride = (long long)I * p->gu_nk * 2 * p->gu_rc;
  p->dn_estride = (long long)H * p->dn_nk * p->dn_rc;
  p->slot_bytes = (int)align_up((size_t)std::max(kCW * 2 * p->gu_rc, kCW * p->dn_rc), 128);
  if (p->tc) {
    p->gu_estride = (long long)(I / 128) * (H / 8) * 4096;
    p->dn_estride = (long long)(H / 128) * (I / 8) * 2048;
    p->slot_bytes = 16384;
  }
  if (p->tq) {
    p->gu_estride = (long long)(I / 128) * (H / 128) * 2 * tq_mat;
    p->dn_estride = (long long)(H / 128) * (I / 128) * tq_mat;
    // FP8: two unit-matrices as they are in HBM; MXFP4: two unit-matrices
    // with each 16-code group in a 16-byte slot, then their scale chunks
    p->slot_bytes = dt == MONO_FP8E4M3_B128 ? (int)(2 * tq_mat) : 2 * 16384 + 2 * 512;
  }

  // grid and shared memory
  // grid: one CTA per SM, a multiple of 4 (the mix partials are read as float4 per output)
  p->G = cfg.grid > 0 ? std::min(cfg.grid, prop.multiProcessorCount) : prop.multiProcessorCount;
  p->G = std::max(4, p->G / 4 * 4);
  p->mix_ctas = p->G;
  p->ymax = (H + p->G - 1) / p->G;
  // region A holds, in turn: the mix_w and hc slices of A2, the mix partials,
  // n [R][H], and the activation rows of the down projections (two halves
  // of at least one row each, for the prefetch of the next expert)
  size_t regA = std::max<size_t>((size_t)RM * H * (cfg.round_bf16 ? 2 : 4), (size_t)RM * I * 4);
  regA = std::max<size_t>(regA, (size_t)2 * I * 4 + 256);
  // prologue staging: the mix_w and residual-stream slices, then at least
  // one row's mix partials of every CTA
  regA = std::max<size_t>(regA, align_up(((size_t)kS * p->ymax * kMixC + (size_t)RM * kS * p->ymax) * 4, 16) +
                                    (size_t)p->G * kMixP * 4);
  if (p->tc || p->tq) {
    regA = std::max<size_t>(regA, (size_t)H * 16);   // n: 8 rows of 16-bit values
    regA = std::max<size_t>(regA, (size_t)I * 32);   // down B: 16 rows (hi/lo of 8 token rows)
  }
  p->regA_bytes = (int)align_up(regA, 128);
  const int smem_max = prop.sharedMemPerBlockOptin;
  SmemLayout L0(0, p->slot_bytes, p->regA_bytes, p->ymax);
  long long room = (long long)smem_max - (long long)L0.ring - 2 * 8 * 16 - kRingGuard;
  // MXFP4 on the tensor cores: each ring slot has its own A scale columns in
  // tensor memory, and there are columns for kF4MaxSlots of them
  p->nst = (int)std::min<long long>(p->tq && dt == MONO_MXFP4 ? kF4MaxSlots : 16, room / p->slot_bytes);
  if (p->nst < 2) {
    std::string m = "shared memory: " + std::to_string(smem_max) + " bytes leave room for " + std::to_string(p->nst) +
                    " ring stages of " + std::to_string(p->slot_bytes) + " bytes (need 2)";
    mono_ffn_destroy(p);
    cudaSetDevice(prev);
    return fail(nullptr, MONO_ERR_INVALID_ARG, m);
  }
  p->smem = (int)SmemLayout(p->nst, p->slot_bytes, p->regA_bytes, p->ymax).total;
  void* kfn = kernel_for(dt, p->tc, p->tq);
  cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, p->smem);
  int occ = 0;
  if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kfn, kThreads, p->smem);
  if (e != cudaSuccess || occ < 1) {
    std::string m = std::string("persistent grid cannot be co-resident: ") +
                    (e != cudaSuccess ? cudaGetErrorString(e) : "occupancy 0");
    mono_ffn_destroy(p);
    cudaSetDevice(prev);
    return fail(nullptr, MONO_ERR_NOT_CORESIDENT, m);
  }

  // storage
  int rc = 0;
  const size_t hc_elem = cfg.hc_dtype == MONO_BF16 ? 2 : 4;
  const size_t norm_elem = cfg.norm_dtype == MONO_BF16 ? 2 : 4;
  p->layers.resize(cfg.n_layers);
  for (auto& l : p->layers) {
    if (!rc) rc = dalloc(p, &l.mix_w, (size_t)kS * H * kMixC * 4, &p->packed_bytes);
    if (!rc) rc = dalloc(p, &l.norm_w, (size_t)H * norm_elem, &p->packed_bytes);
    if (!rc) rc = dalloc(p, &l.router_t, (size_t)E * H * 4, &p->packed_bytes);
    if (!rc) rc = dalloc(p, &l.bias, (size_t)E * 4, &p->packed_bytes);
    if (!rc) rc = dalloc(p, &l.gu, (size_t)(E + 1) * p->gu_estride, &p->packed_bytes);
    if (!rc) rc = dalloc(p, &l.dn, (size_t)(E + 1) * p->dn_estride, &p->packed_bytes);
    if (!rc && p->tq) {
      // FP8: one fp32 block scale per (row, unit); MXFP4: one 512-byte chunk
      // of e8m0 scales per unit-matrix (4 per row)
      const size_t units = (size_t)(E + 1) * (I / 128) * (H / 128);
      rc = dalloc(p, &l.gsc, units * 2 * (dt == MONO_FP8E4M3_B128 ? 128 * 4 : 512), &p->packed_bytes);
      if (!rc) rc = dalloc(p, &l.dsc, units * (dt == MONO_FP8E4M3_B128 ? 128 * 4 : 512), &p->packed_bytes);
      if (!rc && dt == MONO_MXFP4) {
        rc = make_f4_map(p, &l.tm_gu, l.gu, (unsigned long long)units * 2 * 128);
        if (!rc) rc = make_f4_map(p, &l.tm_dn, l.dn, (unsigned long long)units * 128);
      }
    }
  }
  if (!rc) rc = dalloc(p, &p->mix_part, (size_t)p->G * RM * kMixP * 4, &p->scratch_bytes);
  if (!rc) rc = dalloc(p, &p->mix_tot, (size_t)RM * kMixP * 4, &p->scratch_bytes);
  if (!rc) rc = dalloc(p, &p->abuf, (size_t)RM * H * 4, &p->scratch_bytes);
  if (!rc) rc = dalloc(p, &p->sq_part, (size_t)RM * p->G * 4, &p->scratch_bytes);
  if (!rc) rc = dalloc(p, &p->logits, (size_t)RM * E * 4, &p->scratch_bytes);
  if (!rc) rc = dalloc(p, &p->act, (size_t)RM * (K + 1) * I * 4, &p->scratch_bytes);
  if (!rc && (p->tc || p->tq)) rc = dalloc(p, &p->yp, (size_t)RM * (K + 1) * H * 4, &p->scratch_bytes);
  if (!rc && (p->tc || p->tq)) rc = dalloc(p, &p->actb, (size_t)(RM * K + 1) * I * 32, &p->scratch_bytes);
  if (!rc && (p->tc || p->tq)) rc = dalloc(p, &p->gpart, (size_t)p->G * 4 * 128 * 16 * 4, &p->scratch_bytes);
  if (!rc && (p->tc || p->tq)) rc = dalloc(p, &p->dpart, (size_t)p->G * 2 * 128 * 16 * 4, &p->scratch_bytes);
  p->gcnt_n = (size_t)(RM * K + 2) * (I / 128);
  p->dcnt_n = (size_t)(RM * K + 2) * (H / 128);
  if (!rc && (p->tc || p->tq)) rc = dalloc(p, &p->gcnt, p->gcnt_n * 4, &p->scratch_bytes);
  if (!rc && (p->tc || p->tq)) rc = dalloc(p, &p->xready, (size_t)(RM * K + 1) * 4, &p->scratch_bytes);
  if (!rc && (p->tc || p->tq)) rc = dalloc(p, &p->dcnt, p->dcnt_n * 4, &p->scratch_bytes);
  p->pend.assign(cfg.n_layers, nullptr);
  for (int l = 0; l + 1 < cfg.n_layers && !rc; ++l)
    rc = dalloc(p, &p->pend[l], (size_t)RM * (kS + kS * kS + H) * 4, &p->scratch_bytes);
  // residual streams a layer materialises when it opens with a pending
  // expand: the chain's layers alternate between two, a step opened by the
  // attention sublayer's expand uses the first
  if (!rc) rc = dalloc(p, &p->xbuf[0], (size_t)RM * kS * H * hc_elem, &p->scratch_bytes);
  if (cfg.n_layers > 1 && !rc) rc = dalloc(p, &p->xbuf[1], (size_t)RM * kS * H * hc_elem, &p->scratch_bytes);
  if (!rc) rc = dalloc(p, &p->sync, sizeof(SyncBlock) * cfg.n_layers, &p->scratch_bytes);
  if (!rc) rc = dalloc(p, &p->err, sizeof(ErrBlock), &p->scratch_bytes);
  if (!rc) rc = dalloc(p, &p->stage_in, (size_t)RM * kS * H * hc_elem, &p->scratch_bytes);
  if (!rc) rc = dalloc(p, &p->stage_out, (size_t)RM * kS * H * hc_elem, &p->scratch_bytes);
  if (!rc) {
    cudaMemset(p->sync, 0, sizeof(SyncBlock) * cfg.n_layers);
    cudaMemset(p->err, 0, sizeof(ErrBlock));
    cudaMemset(p->act, 0, (size_t)RM * (K + 1) * I * 4);
    if (p->tc || p->tq) {
      cudaMemset(p->yp, 0, (size_t)RM * (K + 1) * H * 4);
      cudaMemset(p->gcnt, 0, p->gcnt_n * 4);
      cudaMemset(p->dcnt, 0, p->dcnt_n * 4);
      cudaMemset(p->xready, 0, (size_t)(RM * K + 1) * 4);
    }
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) rc = cuda_fail(p, e, "plan setup");
  }
  if (rc) {
    std::string m = p->last_error;
    mono_ffn_destroy(p);
    cudaSetDevice(prev);
    return fail(nullptr, rc, m);
  }
  cudaSetDevice(prev);
  *out = p;
  return MONO_OK;
}

extern "C" int mono_ffn_pack_weights(mono_ffn_plan_t* p, int layer, const mono_ffn_layer_weights* w, void* stream) {
  if (!p) return fail(nullptr, MONO_ERR_INVALID_ARG, "pack: NULL plan");
  if (!w || layer < 0 || layer >= p->cfg.n_layers) return fail(p, MONO_ERR_INVALID_ARG, "pack: bad layer or weights");
  std::string why;
  if (!w->mix_w) why += "mix_w is NULL\n";
  if (!w->norm_w) why += "norm_w is NULL\n";
  if (!w->router_w && !p->cfg.dense) why += "router_w is NULL\n";
  if (!w->router_bias && !p->cfg.dense) why += "router_bias is NULL\n";
  if (!w->w_gate || !w->w_up || !w->w_down) why += "expert weights are NULL\n";
  if (!why.empty()) return fail(p, MONO_ERR_INVALID_ARG, why);
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(p->cfg.device);
  cudaStream_t st = (cudaStream_t)stream;
  const int H = p->cfg.hidden, I = p->cfg.inter, E = p->cfg.n_routed;
  LayerSlot& l = p->layers[layer];
  const size_t norm_elem = p->cfg.norm_dtype == MONO_BF16 ? 2 : 4;
  cudaMemcpyAsync(l.mix_w, w->mix_w, (size_t)kS * H * kMixC * 4, cudaMemcpyDeviceToDevice, st);
  cudaMemcpyAsync(l.norm_w, w->norm_w, (size_t)H * norm_elem, cudaMemcpyDeviceToDevice, st);
  if (!p->cfg.dense) {   // a dense layer has no router
    cudaMemcpyAsync(l.bias, w->router_bias, (size_t)E * 4, cudaMemcpyDeviceToDevice, st);
    transpose_f32_kernel<<<dim3((E + 31) / 32, (H + 31) / 32), dim3(32, 8), 0, st>>>(w->router_w, l.router_t, H, E);
  }
  int rc = 0;
  if (p->tc) {
    // 128-row blocks of core matrices: gate and up of a rowgroup side by
    // side, down in its own blocks
    const int th = 256;
    auto grid = [&](long long n) { return (unsigned)std::min<long long>((n + th - 1) / th, 148LL * 64); };
    const long long n_gu = (long long)(E + 1) * I * (H / 8), n_dn = (long long)(E + 1) * H * (I / 8);
    pack_tc_kernel<<<grid(n_gu), th, 0, st>>>((const uint16_t*)w->w_gate, l.gu, E + 1, I, H, 256, 0);
    pack_tc_kernel<<<grid(n_gu), th, 0, st>>>((const uint16_t*)w->w_up, l.gu, E + 1, I, H, 256, 128);
    pack_tc_kernel<<<grid(n_dn), th, 0, st>>>((const uint16_t*)w->w_down, l.dn, E + 1, H, I, 128, 0);
    cudaError_t e2 = cudaGetLastError();
    cudaSetDevice(prev);
    if (e2 != cudaSuccess) return cuda_fail(p, e2, "pack");
    l.packed = true;
    return MONO_OK;
  }
  if (p->tq) {
    const bool fp8 = p->wt == W_FP8;
    const int th = 256;
    auto grid = [&](long long n) { return (unsigned)std::min<long long>((n + th - 1) / th, 148LL * 64); };
    const long long mat = 16384;   // FP8: one unit-matrix
    const int ub = 128;            // FP8: unit-row bytes of codes
    const int gu_rb = fp8 ? H : H / 2, dn_rb = fp8 ? I : I / 2;    // code bytes per weight row
    if (!fp8) {
      // e8m0 code 255 is NaN: not a scale the tensor-core path can expand
      unsigned int* mm = nullptr;
      cudaError_t ea = cudaMalloc(&mm, 8);
      if (ea != cudaSuccess) {
        cudaSetDevice(prev);
        return cuda_fail(p, ea, "pack: scale range scratch");
      }
      const unsigned int init[2] = {255u, 0u};
      cudaMemcpyAsync(mm, init, 8, cudaMemcpyHostToDevice, st);
      byte_range_kernel<<<148, 256, 0, st>>>((const uint8_t*)w->s_gate, (long long)(E + 1) * I * (H / 32), mm);
      byte_range_kernel<<<148, 256, 0, st>>>((const uint8_t*)w->s_up, (long long)(E + 1) * I * (H / 32), mm);
      byte_range_kernel<<<148, 256, 0, st>>>((const uint8_t*)w->s_down, (long long)(E + 1) * H * (I / 32), mm);
      unsigned int got[2] = {0u, 0u};
      cudaMemcpyAsync(got, mm, 8, cudaMemcpyDeviceToHost, st);
      ea = cudaStreamSynchronize(st);
      cudaFree(mm);
      if (ea != cudaSuccess) {
        cudaSetDevice(prev);
        return cuda_fail(p, ea, "pack: scale range");
      }
      if (got[1] > 254u) {
        cudaSetDevice(prev);
        return fail(p, MONO_ERR_INVALID_ARG, "pack: MXFP4 scale code 255 (NaN)");
      }
    }
    if (fp8) {
      pack_tq_codes_kernel<<<grid((long long)(E + 1) * I * (gu_rb / 16)), th, 0, st>>>(
          (const uint8_t*)w->w_gate, l.gu, E + 1, I, gu_rb, ub, 2 * mat, 0);
      pack_tq_codes_kernel<<<grid((long long)(E + 1) * I * (gu_rb / 16)), th, 0, st>>>(
          (const uint8_t*)w->w_up, l.gu, E + 1, I, gu_rb, ub, 2 * mat, (int)mat);
      pack_tq_codes_kernel<<<grid((long long)(E + 1) * H * (dn_rb / 16)), th, 0, st>>>(
          (const uint8_t*)w->w_down, l.dn, E + 1, H, dn_rb, ub, mat, 0);
      pack_tq_scales_kernel<<<grid((long long)(E + 1) * I * (H / 128)), th, 0, st>>>(
          (const float*)w->s_gate, l.gsc, E + 1, I, H / 128, 2, 0);
      pack_tq_scales_kernel<<<grid((long long)(E + 1) * I * (H / 128)), th, 0, st>>>(
          (const float*)w->s_up, l.gsc, E + 1, I, H / 128, 2, 1);
      pack_tq_scales_kernel<<<grid((long long)(E + 1) * H * (I / 128)), th, 0, st>>>(
          (const float*)w->s_down, l.dsc, E + 1, H, I / 128, 1, 0);
    } else {
      // unit-matrices of 128 rows x 64 bytes (gate/up as pairs), and their
      // 512-byte scale chunks in the order the tensor memory copy takes
      pack_mx_codes_kernel<<<grid((long long)(E + 1) * I * (H / 128) * 4), th, 0, st>>>(
          (const uint8_t*)w->w_gate, l.gu, E + 1, I, H / 2, 2, 0);
      pack_mx_codes_kernel<<<grid((long long)(E + 1) * I * (H / 128) * 4), th, 0, st>>>(
          (const uint8_t*)w->w_up, l.gu, E + 1, I, H / 2, 2, 1);
      pack_mx_codes_kernel<<<grid((long long)(E + 1) * H * (I / 128) * 4), th, 0, st>>>(
          (const uint8_t*)w->w_down, l.dn, E + 1, H, I / 2, 1, 0);
      uint8_t* gsc = reinterpret_cast<uint8_t*>(l.gsc);
      uint8_t* dsc = reinterpret_cast<uint8_t*>(l.dsc);
      pack_mx_scales_kernel<<<grid((long long)(E + 1) * I * (H / 32)), th, 0, st>>>(
          (const uint8_t*)w->s_gate, gsc, E + 1, I, H / 32, 2, 0);
      pack_mx_scales_kernel<<<grid((long long)(E + 1) * I * (H / 32)), th, 0, st>>>(
          (const uint8_t*)w->s_up, gsc, E + 1, I, H / 32, 2, 1);
      pack_mx_scales_kernel<<<grid((long long)(E + 1) * H * (I / 32)), th, 0, st>>>(
          (const uint8_t*)w->s_down, dsc, E + 1, H, I / 32, 1, 0);
    }
    cudaError_t e2 = cudaGetLastError();
    cudaSetDevice(prev);
    if (e2 != cudaSuccess) return cuda_fail(p, e2, "pack");
    l.packed = true;
    return MONO_OK;
  }
  // gate and up share an item: [gate chunk | up chunk]
  rc = pack_matrix(p, w->w_gate, w->s_gate, l.gu, (long long)(E + 1) * I, H, p->gu_kc, p->gu_nk, p->gu_rc,
                   2 * p->gu_rc, 0, st);
  if (!rc)
    rc = pack_matrix(p, w->w_up, w->s_up, l.gu, (long long)(E + 1) * I, H, p->gu_kc, p->gu_nk, p->gu_rc, 2 * p->gu_rc,
                     p->gu_rc, st);
  if (!rc)
    rc = pack_matrix(p, w->w_down, w->s_down, l.dn, (long long)(E + 1) * H, I, p->dn_kc, p->dn_nk, p->dn_rc, p->dn_rc,
                     0, st);
  cudaError_t e = cudaGetLastError();
  cudaSetDevice(prev);
  if (rc) return rc;
  if (e != cudaSuccess) return cuda_fail(p, e, "pack");
  l.packed = true;
  return MONO_OK;
}

extern "C" int mono_ffn_set_taps(mono_ffn_plan_t* p, int layer, const mono_ffn_taps* t) {
  if (!p) return fail(nullptr, MONO_ERR_INVALID_ARG, "set_taps: NULL plan");
  if (layer < 0 || layer >= p->cfg.n_layers) return fail(p, MONO_ERR_INVALID_ARG, "set_taps: bad layer");
  Taps& d = p->layers[layer].taps;
  if (!t) {
    d = Taps{};
    return MONO_OK;
  }
  d.mix = t->mix;
  d.pre = t->pre;
  d.post = t->post;
  d.comb = t->comb;
  d.n = t->n;
  d.logits = t->logits;
  d.idx = t->idx;
  d.w = t->w;
  d.y = t->y;
  d.x = t->x;
  return MONO_OK;
}

namespace {

// The attention sublayer's pending post / expand that a step may open with
// (mono_ffn_step_pending); all NULL for a plain step.
struct Pending {
  const void* x;
  const float* post;
  const float* comb;
  const void* y;
};

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const char* x = (const char*)a;
  const char* y = (const char*)b;
  return x < y + nb && y < x + na;
}

int step_impl(mono_ffn_plan_t* p, int rows, const void* hc_in, const Pending* pd, const int* row_slot, void* hc_out,
              void* stream);

}  // namespace

extern "C" int mono_ffn_step(mono_ffn_plan_t* p, int rows, const void* hc_in, void* hc_out, void* stream) {
  if (!p) return fail(nullptr, MONO_ERR_INVALID_ARG, "step: NULL plan");
  if (rows == 0) return MONO_OK;
  if (rows < 0 || rows > p->cfg.max_rows)
    return fail(p, MONO_ERR_INVALID_ARG, "step: rows " + std::to_string(rows) + " outside [0, max_rows = " +
                                             std::to_string(p->cfg.max_rows) + "]");
  if (!hc_in || !hc_out) return fail(p, MONO_ERR_INVALID_ARG, "step: NULL hc_in or hc_out");
  const size_t hc_bytes = (size_t)rows * kS * p->cfg.hidden * (p->cfg.hc_dtype == MONO_BF16 ? 2 : 4);
  if (overlaps(hc_in, hc_bytes, hc_out, hc_bytes)) return fail(p, MONO_ERR_INVALID_ARG, "step: hc_in and hc_out overlap");
  return step_impl(p, rows, hc_in, nullptr, nullptr, hc_out, stream);
}

extern "C" int mono_ffn_step_padded(mono_ffn_plan_t* p, int width, const int* row_slot, const void* hc_in,
                                    void* hc_out, void* stream) {
  if (!p) return fail(nullptr, MONO_ERR_INVALID_ARG, "step_padded: NULL plan");
  if (width == 0) return MONO_OK;
  if (width < 0 || width > p->cfg.max_rows)
    return fail(p, MONO_ERR_INVALID_ARG, "step_padded: width " + std::to_string(width) + " outside [0, max_rows = " +
                                             std::to_string(p->cfg.max_rows) + "]");
  if (!row_slot || !hc_in || !hc_out) return fail(p, MONO_ERR_INVALID_ARG, "step_padded: NULL argument");
  const size_t hc_bytes = (size_t)width * kS * p->cfg.hidden * (p->cfg.hc_dtype == MONO_BF16 ? 2 : 4);
  if (overlaps(hc_in, hc_bytes, hc_out, hc_bytes))
    return fail(p, MONO_ERR_INVALID_ARG, "step_padded: hc_in and hc_out overlap");
  return step_impl(p, width, hc_in, nullptr, row_slot, hc_out, stream);
}

extern "C" int mono_ffn_step_pending(mono_ffn_plan_t* p, int rows, const void* x_attn, const float* attn_post,
                                     const float* attn_comb, const void* y_attn, void* hc_out, void* stream) {
  if (!p) return fail(nullptr, MONO_ERR_INVALID_ARG, "step_pending: NULL plan");
  if (rows == 0) return MONO_OK;
  if (rows < 0 || rows > p->cfg.max_rows)
    return fail(p, MONO_ERR_INVALID_ARG, "step_pending: rows " + std::to_string(rows) + " outside [0, max_rows = " +
                                             std::to_string(p->cfg.max_rows) + "]");
  if (!x_attn || !attn_post || !attn_comb || !y_attn || !hc_out)
    return fail(p, MONO_ERR_INVALID_ARG, "step_pending: NULL argument");
  const size_t el = p->cfg.hc_dtype == MONO_BF16 ? 2 : 4;
  const size_t hc_bytes = (size_t)rows * kS * p->cfg.hidden * el, y_bytes = (size_t)rows * p->cfg.hidden * el;
  std::string why;
  if (overlaps(x_attn, hc_bytes, hc_out, hc_bytes)) why += "x_attn and hc_out overlap\n";
  if (overlaps(y_attn, y_bytes, hc_out, hc_bytes)) why += "y_attn and hc_out overlap\n";
  if (overlaps(attn_post, (size_t)rows * kS * 4, hc_out, hc_bytes) ||
      overlaps(attn_comb, (size_t)rows * kS * kS * 4, hc_out, hc_bytes))
    why += "attn_post or attn_comb overlaps hc_out\n";
  if (!why.empty()) return fail(p, MONO_ERR_INVALID_ARG, "step_pending: " + why);
  const Pending pd{x_attn, attn_post, attn_comb, y_attn};
  return step_impl(p, rows, x_attn, &pd, nullptr, hc_out, stream);
}

namespace {

int step_impl(mono_ffn_plan_t* p, int rows, const void* hc_in, const Pending* pd, const int* row_slot, void* hc_out,
              void* stream) {
  for (int l = 0; l < p->cfg.n_layers; ++l)
    if (!p->layers[l].packed)
      return fail(p, MONO_ERR_NOT_PACKED, "step: layer " + std::to_string(l) + " has no packed weights");
  int prev = 0;
  cudaGetDevice(&prev);
  if (prev != p->cfg.device) cudaSetDevice(p->cfg.device);
  const int L = p->cfg.n_layers;
  void* kfn = kernel_for(p->wt, p->tc, p->tq);
  cudaError_t e = cudaSuccess;
  for (int l = 0; l < L && e == cudaSuccess; ++l) {
    const LayerSlot& ls = p->layers[l];
    Params prm{};
    prm.H = p->cfg.hidden;
    prm.I = p->cfg.inter;
    prm.E = p->cfg.n_routed;
    prm.K = p->cfg.top_k;
    prm.R = rows;
    prm.G = p->G;
    prm.layer = l;
    prm.first = l == 0 && !pd;
    prm.dense = p->cfg.dense;
    prm.mx8 = p->cfg.act_mx8;
    prm.last = l == L - 1;
    prm.mix_ctas = p->mix_ctas;
    prm.hc_bf16 = p->cfg.hc_dtype == MONO_BF16;
    prm.norm_bf16 = p->cfg.norm_dtype == MONO_BF16;
    prm.round_bf16 = p->cfg.round_bf16 != 0;
    prm.rms_eps = p->cfg.rms_eps;
    prm.pre_eps = p->cfg.pre_eps;
    prm.post_mult = p->cfg.post_mult;
    prm.route_scale = p->cfg.route_scale;
    prm.denom_clamp = p->cfg.denom_clamp;
    prm.sink_iters = p->cfg.sinkhorn_iters;
    // layer l reads the residual streams of layer l - 1 (hc_in for layer 0,
    // or, opened by a pending expand, the attention sublayer's input) and
    // materialises its own in xbuf[l % 2] when it opens with an expand
    prm.x_prev = l == 0 ? hc_in : l == 1 ? (pd ? p->xbuf[0] : hc_in) : p->xbuf[(l - 1) % 2];
    prm.xbuf = prm.first ? nullptr : p->xbuf[l % 2];
    prm.hc_out = hc_out;
    if (l > 0) {
      prm.pend_post = p->pend[l - 1];
      prm.pend_comb = p->pend[l - 1] + rows * kS;
      prm.pend_y = p->pend[l - 1] + rows * kS + rows * kS * kS;
      prm.pend_y_bf16 = 0;
    } else if (pd) {
      prm.pend_post = pd->post;
      prm.pend_comb = pd->comb;
      prm.pend_y = pd->y;
      prm.pend_y_bf16 = p->cfg.hc_dtype == MONO_BF16;
    }
    prm.pend_out = l + 1 < L ? p->pend[l] : nullptr;
    prm.mix_w = ls.mix_w;
    prm.norm_w = ls.norm_w;
    prm.router_t = ls.router_t;
    prm.bias = ls.bias;
    prm.gu = ls.gu;
    prm.dn = ls.dn;
    prm.gu_kc = p->gu_kc;
    prm.gu_nk = p->gu_nk;
    prm.gu_rc = p->gu_rc;
    prm.dn_kc = p->dn_kc;
    prm.dn_nk = p->dn_nk;
    prm.dn_rc = p->dn_rc;
    prm.gu_estride = p->gu_estride;
    prm.dn_estride = p->dn_estride;
    prm.mix_part = p->mix_part;
    prm.mix_tot = p->mix_tot;
    prm.abuf = p->abuf;
    prm.sq_part = p->sq_part;
    prm.logits = p->logits;
    prm.act = p->act;
    prm.yp = p->yp;
    prm.actb = p->actb;
    prm.gpart = p->gpart;
    prm.dpart = p->dpart;
    prm.gcnt = p->gcnt;
    prm.dcnt = p->dcnt;
    prm.xready = p->xready;
    prm.gsc = ls.gsc;
    prm.dsc = ls.dsc;
    prm.tm_gu = ls.tm_gu;
    prm.tm_dn = ls.tm_dn;
    prm.n_xready = p->xready ? rows * p->cfg.top_k + 1 : 0;
    prm.n_xready_all = p->xready ? p->cfg.max_rows * p->cfg.top_k + 1 : 0;
    prm.sync = p->sync + l;
    prm.err = p->err;
    prm.taps = ls.taps;
    prm.nst = p->nst;
    prm.slot_bytes = p->slot_bytes;
    prm.regA_bytes = p->regA_bytes;
    prm.ymax = p->ymax;
    prm.timeout_ns = (unsigned long long)p->cfg.wait_timeout_us * 1000ull;
    prm.row_slot = row_slot;
    prm.fault_cta = p->fault_cta;
    prm.fault_stage = p->fault_cta >= 0 ? p->fault_stage : 0;
    prm.jitter_ns = p->jitter_ns;
    prm.trace = p->trace ? p->trace + (size_t)l * p->G * kTracePoints : nullptr;

    cudaLaunchConfig_t lc{};
    lc.gridDim = dim3(p->G);
    lc.blockDim = dim3(kThreads);
    lc.dynamicSmemBytes = p->smem;
    lc.stream = (cudaStream_t)stream;
    // cooperative: every CTA resident at once (the grid-wide stages wait on
    // one another); a chain's later layers also as programmatic dependent
    // launches, so that each starts launching while the layer before it ends
    // (the kernel waits for that layer before it reads anything)
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = (l > 0 && p->pdl_ok) ? 2 : 1;
    void* args[] = {&prm};
    e = cudaLaunchKernelExC(&lc, kfn, args);
    if (e != cudaSuccess && lc.numAttrs == 2) {
      // the driver refused the combination: launch as before from now on
      cudaGetLastError();
      p->pdl_ok = false;
      lc.numAttrs = 1;
      e = cudaLaunchKernelExC(&lc, kfn, args);
    }
  }
  if (prev != p->cfg.device) cudaSetDevice(prev);
  if (e != cudaSuccess) return cuda_fail(p, e, "step launch");
  return MONO_OK;
}

}  // namespace

extern "C" int mono_ffn_step_host(mono_ffn_plan_t* p, int rows, const void* hc_in_host, void* hc_out_host,
                                  void* stream) {
  if (!p) return fail(nullptr, MONO_ERR_INVALID_ARG, "step_host: NULL plan");
  if (rows == 0) return MONO_OK;
  if (rows < 0 || rows > p->cfg.max_rows) return fail(p, MONO_ERR_INVALID_ARG, "step_host: rows out of range");
  if (!hc_in_host || !hc_out_host) return fail(p, MONO_ERR_INVALID_ARG, "step_host: NULL buffer");
  const size_t bytes = (size_t)rows * kS * p->cfg.hidden * (p->cfg.hc_dtype == MONO_BF16 ? 2 : 4);
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(p->cfg.device);
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(p->stage_in, hc_in_host, bytes, cudaMemcpyHostToDevice, st);
  int rc = e == cudaSuccess ? mono_ffn_step(p, rows, p->stage_in, p->stage_out, stream) : cuda_fail(p, e, "H2D");
  if (!rc) {
    e = cudaMemcpyAsync(hc_out_host, p->stage_out, bytes, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) rc = cuda_fail(p, e, "D2H");
  }
  cudaSetDevice(prev);
  return rc;
}

extern "C" int mono_ffn_query_error(mono_ffn_plan_t* p, mono_ffn_status* st) {
  if (!p) return fail(nullptr, MONO_ERR_INVALID_ARG, "query_error: NULL plan");
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(p->cfg.device);
  ErrBlock eb{};
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&eb, p->err, sizeof(eb), cudaMemcpyDeviceToHost);
  int rc = MONO_OK;
  if (e != cudaSuccess) {
    rc = cuda_fail(p, e, "query_error");
  } else if (eb.code || eb.abort) {
    rc = eb.code == 7u ? MONO_ERR_DEVICE_TIMEOUT : MONO_ERR_DEVICE_ABORTED;
    p->last_error = "device wait failed: stage " + std::to_string(eb.stage) + ", cta " + std::to_string(eb.cta) +
                    ", layer " + std::to_string(eb.layer);
    // reset the sync state so the next step starts clean
    cudaMemset(p->sync, 0, sizeof(SyncBlock) * p->cfg.n_layers);
    cudaMemset(p->err, 0, sizeof(ErrBlock));
    if (p->gcnt) cudaMemset(p->gcnt, 0, p->gcnt_n * 4);
    if (p->dcnt) cudaMemset(p->dcnt, 0, p->dcnt_n * 4);
    if (p->xready) cudaMemset(p->xready, 0, (size_t)(p->cfg.max_rows * p->cfg.top_k + 1) * 4);
    cudaDeviceSynchronize();
  }
  if (st) {
    st->code = rc == MONO_ERR_DEVICE_TIMEOUT || rc == MONO_ERR_DEVICE_ABORTED ? rc : 0;
    st->stage = (int)eb.stage;
    st->cta = (int)eb.cta;
    st->layer = (int)eb.layer;
  }
  cudaSetDevice(prev);
  return rc;
}

extern "C" int mono_ffn_get_info(const mono_ffn_plan_t* p, mono_ffn_info* info) {
  if (!p || !info) return MONO_ERR_INVALID_ARG;
  const int H = p->cfg.hidden, E = p->cfg.n_routed;
  info->grid = p->G;
  info->threads = kThreads;
  info->smem_bytes = p->smem;
  info->ring_stages = p->nst;
  info->ring_slot_bytes = p->slot_bytes;
  info->expert_bytes = p->gu_estride + p->dn_estride;
  if (p->tq && p->wt == W_FP8)   // the FP8 block scales travel in their own arrays
    info->expert_bytes += (int64_t)(p->cfg.inter / 128) * (H / 128) * 256 * 4 + (int64_t)(H / 128) * (p->cfg.inter / 128) * 128 * 4;
  if (p->tq && p->wt == W_FP4)   // and the MXFP4 e8m0 block scales (one byte per 32 codes)
    info->expert_bytes += (int64_t)(p->cfg.inter / 128) * (H / 128) * 3 * 512;
  info->dense_bytes = (int64_t)kS * H * kMixC * 4 + (p->cfg.dense ? 0 : (int64_t)E * H * 4 + (int64_t)E * 4) +
                      (int64_t)H * (p->cfg.norm_dtype == MONO_BF16 ? 2 : 4);
  info->packed_bytes = p->packed_bytes;
  info->scratch_bytes = p->scratch_bytes;
  return MONO_OK;
}

extern "C" int mono_ffn_set_trace(mono_ffn_plan_t* p, unsigned long long* buf) {
  if (!p) return MONO_ERR_INVALID_ARG;
  p->trace = buf;
  return MONO_OK;
}

extern "C" int mono_ffn_debug_skip_arrival(mono_ffn_plan_t* p, int cta, int stage) {
  if (!p) return fail(nullptr, MONO_ERR_INVALID_ARG, "debug_skip_arrival: NULL plan");
  if (cta < 0) {
    p->fault_cta = -1;
    p->fault_stage = 0;
    return MONO_OK;
  }
  const bool known = stage == MONO_STAGE_MIX || stage == MONO_STAGE_LOGITS || stage == MONO_STAGE_ACT ||
                     stage == MONO_STAGE_Y || stage == MONO_STAGE_COLLAPSE;
  if (!known || cta >= p->G)
    return fail(p, MONO_ERR_INVALID_ARG, "debug_skip_arrival: cta must be < grid and stage one of MIX, LOGITS, "
                                         "ACT, Y, COLLAPSE");
  if (stage == MONO_STAGE_Y && !(p->tc || p->tq))
    return fail(p, MONO_ERR_INVALID_ARG, "debug_skip_arrival: the CUDA-core kernel has no Y stage");
  p->fault_cta = cta;
  p->fault_stage = stage;
  return MONO_OK;
}

extern "C" int mono_ffn_debug_jitter(mono_ffn_plan_t* p, unsigned max_ns) {
  if (!p) return fail(nullptr, MONO_ERR_INVALID_ARG, "debug_jitter: NULL plan");
  if (max_ns > 100000u) return fail(p, MONO_ERR_INVALID_ARG, "debug_jitter: max_ns above 100000");
  p->jitter_ns = max_ns;
  return MONO_OK;
}

#include "route_noalloc.cuh"
