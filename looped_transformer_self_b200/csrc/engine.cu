// Step engine and C ABI of the pipelined self-speculative decoder.
//
// One decode step = one CUDA-graph replay of: embedding (+ prelude layers) for
// branches opened in the last step, every shared-block layer once over all
// active rows at their own depths, readouts (coda, final norm, LM head,
// temperature / top-p) for rows at proposal depths and at R, the accept /
// proposal kernel and the bookkeeping kernel.  No host round trip inside a
// step; the host only reads the committed count between batches of steps.
// ("LoopSpec", liuzhao09.github.io/papers/loopspec.html, sections 2.2-2.4;
// section 2.4 notes that batching needs CUDA graphs that include the cache
// index updates -- here one fixed-capacity graph covers every batch size,
// since the row count lives on the device.)
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <string>
#include <vector>

#include "../../include/looped_spec.h"
#include "decide.cuh"
#include "gemm.cuh"
#include "layers.cuh"

namespace lt {

struct LayerW {
  const void *g1, *wqkv, *wo, *g2, *wgu, *wd;
  GemmOperand tm_qkv, tm_o, tm_gu, tm_d;          // hi parts (or the bf16 weights)
  GemmOperand tm_qkv_lo, tm_o_lo, tm_gu_lo, tm_d_lo;  // lo parts (split tf32 only)
};

struct Handle {
  lt_model_config m;
  lt_decode_config dc;
  bool f32 = false;
  int mode = 0;          // GEMM mode: 0 bf16, 2 split tf32 (fp32 models)
  size_t lo_d = 0, lo_f = 0;  // lo-plane offsets of the fp32 operand buffers
  float* wsplit = nullptr;    // hi / lo copies of fp32 GEMM weights
  size_t wsplit_elems = 0;
  int C = 0, S = 0, max_splits = 0, n_tags = 0, planes = 0, max_pos = 0;
  int tags[3] = {0, 0, 0};
  cudaStream_t stream = nullptr;
  char* ws = nullptr;
  size_t ws_bytes = 0;
  Dev D;
  float *h = nullptr, *hc = nullptr, *q = nullptr, *attn_part = nullptr, *part = nullptr;
  int* attn_cnt = nullptr;  // per (row, head) split-arrival counters (kept at zero between uses)
  const int* lists_override = nullptr;  // caller slot lists of lt_block_pass
  cudaGraphExec_t pass_graph = nullptr;
  int pass_graph_rows = -1;
  float* ssq = nullptr;     // [ceil(d/128)][C] sum-of-squares parts of the pending RMSNorm
  int ssq_tiles = 0;
  unsigned long long *cnt_o = nullptr, *cnt_gu = nullptr, *cnt_d = nullptr;  // epilogue arrivals
  int *need_o = nullptr, *need_gu = nullptr, *need_d = nullptr;  // arrivals completing a group
  void *Xd = nullptr, *Xo = nullptr, *Xf = nullptr, *kv = nullptr;
  float2* rope = nullptr;
  int* gemm_tab = nullptr;
  std::vector<int> plane_base;
  GemmShape sh_qkv, sh_o, sh_gu, sh_d, sh_head;
  GemmOperand tm_Xd, tm_Xo, tm_Xf, tm_head;
  GemmOperand tm_Xd_lo, tm_Xo_lo, tm_Xf_lo, tm_head_lo;
  const void *embed = nullptr, *final_norm = nullptr, *head = nullptr;
  std::vector<LayerW> layers;
  bool loaded = false, prefilled = false, begun = false;
  int P = 0;
  cudaGraphExec_t graph = nullptr;
  bool use_pdl = true, use_graph = true;
  int kernels_per_step = 0;  // launches counted while capturing the step graph
  bool counting = false;
  // profiling: events around GEMMs and attention of un-graphed steps
  bool profiling = false;
  int prof_cat = 0;  // 0: shared-block layer, 1: prelude / coda / head
  struct Ev {
    int kind;  // 0 gemm core, 1 gemm other, 2 attention
    int gate;  // device flag that lets the launch work: 0 none, 1 run, 2 new rows, 3 readouts
    double bytes;
    cudaEvent_t a, b;
  };
  std::vector<Ev> evs;
  std::string err;
};

// Records an event pair around one launch when profiling.
struct ProfScope {
  Handle* H;
  int idx = -1;
  ProfScope(Handle* h, int kind, double bytes, int gate = 0) : H(h) {
    if (!H->profiling) return;
    Handle::Ev e;
    e.kind = kind;
    e.gate = gate;
    e.bytes = bytes;
    cudaEventCreate(&e.a);
    cudaEventCreate(&e.b);
    cudaEventRecord(e.a, H->stream);
    H->evs.push_back(e);
    idx = (int)H->evs.size() - 1;
  }
  ~ProfScope() {
    if (idx >= 0) cudaEventRecord(H->evs[idx].b, H->stream);
  }
};

static int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

constexpr int kMaxDev = 64;
static int cur_dev() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev >= 0 && dev < kMaxDev ? dev : 0;
}

static int* g_launch_counter = nullptr;  // set while the step graph is captured

template <typename... KArgs, typename... Args>
static cudaError_t launch(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block,
                          cudaStream_t st, Args&&... args) {
  if (g_launch_counter) ++*g_launch_counter;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// A 1024-thread kernel on clusters of RO_CL CTAs along x (one cluster per row).
template <typename... KArgs, typename... Args>
static cudaError_t launch_cluster(Handle* H, void (*kern)(KArgs...), dim3 grid, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(1024);
  cfg.stream = H->stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = RO_CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = H->use_pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// workspace layout
// ---------------------------------------------------------------------------
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(char* b) : base(b) {}
  template <typename T>
  T* take(size_t n) {
    off = (off + 255) & ~(size_t)255;
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += n * sizeof(T);
    return p;
  }
};

static int validate(const lt_model_config* m, const lt_decode_config* dc, std::string* why) {
  auto bad = [&](const char* s) {
    if (why) *why = s;
    return LT_ERR_SHAPE;
  };
  if (!m || !dc) return LT_ERR_ARG;
  if (m->dtype != LT_F32 && m->dtype != LT_BF16) return bad("dtype must be LT_F32 or LT_BF16");
  if (m->d_model <= 0 || m->n_heads <= 0 || m->head_dim <= 0 || m->ffn <= 0 || m->vocab <= 0)
    return bad("non-positive model size");
  if (m->n_heads * m->head_dim != m->d_model) return bad("n_heads * head_dim != d_model");
  if (m->head_dim != 32 && m->head_dim != 64 && m->head_dim != 96 && m->head_dim != 128)
    return bad("head_dim must be 32, 64, 96 or 128");
  if (m->R < 1 || m->R > 32) return bad("R must be in 1..32");
  if (m->n_core < 1 || m->n_prelude < 0 || m->n_coda < 0) return bad("layer counts");
  const int esz = m->dtype == LT_F32 ? 4 : 2;
  if ((m->d_model * esz) % 16 || (m->ffn * esz) % 16) return bad("d_model/ffn rows must be 16-byte multiples");
  if (m->ffn % 128) return bad("ffn must be a multiple of 128 (SwiGLU tiles pair gate with up)");
  const int C = dc->max_branches;
  if (C != 8 && C != 16 && C != 32 && C != 64) return bad("max_branches must be 8, 16, 32 or 64");
  if (dc->d1 < 0 || dc->d1 >= m->R || dc->d2 < 0 || (dc->d2 && (dc->d2 <= dc->d1 || dc->d2 >= m->R)))
    return bad("need 1 <= d1 < d2 < R (d2 = 0: single proposal)");
  if (dc->max_ctx < 2) return bad("max_ctx");
  if (dc->max_ctx + C + 8 > (1 << 24)) return bad("max_ctx too large");
  if (dc->temperature < 0.f || !(dc->top_p > 0.f) || dc->top_p > 1.f) return bad("temperature/top_p");
  if (dc->second_mode < 0 || dc->second_mode > 2) return bad("second_mode");
  if (dc->copy_k < 0 || (dc->copy_k > 0 && (dc->copy_max_len < 1 || dc->copy_max_len > CPMAX ||
                                            dc->copy_match_cap < dc->copy_k ||
                                            dc->copy_reserve < 0 || !(dc->copy_tau >= 0.f))))
    return bad("copy proposals: need copy_k <= copy_match_cap, 1 <= copy_max_len <= 32, copy_reserve >= 0, copy_tau >= 0");
  if (dc->copy_k > 0 && dc->d1 < 1) return bad("copy proposals need d1 >= 1");
  return LT_OK;
}

static size_t carve(Handle* H, char* base) {
  const lt_model_config& m = H->m;
  const int C = H->C, d = m.d_model, V = m.vocab, f = m.ffn;
  const size_t esz = H->f32 ? 4 : 2;
  Carver cv(base);
  Dev& D = H->D;
  D.ctl = cv.take<Ctl>(1);
  int** tab[] = {&D.b_alive, &D.b_uid, &D.b_parent, &D.b_slot, &D.b_pos, &D.b_tok, &D.b_depth,
                 &D.b_x1, &D.b_x2, &D.b_gate, &D.b_c1, &D.b_c2};
  for (int** p : tab) *p = cv.take<int>(C);
  D.b_chain = cv.take<int>((size_t)C * WIN);
  int** cps[] = {&D.b_copy, &D.b_crow, &D.cp_fail, &D.cp_len, &D.v_tok, &D.v_src, &D.v_fb};
  for (int** p : cps) *p = cv.take<int>(C);
  D.cp_tok = cv.take<int>((size_t)C * CPMAX);
  int** rows[] = {&D.r_tok, &D.r_pos, &D.r_slot, &D.r_depth, &D.r_ro, &D.r_blen, &D.r_boff,
                  &D.m_alive, &D.m_new, &D.m_ro};
  for (int** p : rows) *p = cv.take<int>(C);
  D.lists = cv.take<int>(H->dc.max_ctx);
  D.committed = cv.take<int>(H->dc.max_ctx);
  D.slot_bits = cv.take<unsigned int>((H->S + 31) / 32);
  D.log_tok = cv.take<int>(H->dc.max_ctx);
  D.log_src = cv.take<int>(H->dc.max_ctx);
  D.log_step = cv.take<int>(H->dc.max_ctx);
  D.trace = cv.take<int>((size_t)std::max(1, H->dc.trace_steps) * C * 4);
  D.ro_arg = cv.take<int>(C);
  const int gc = sm_count();
  GemmShape* shapes[] = {&H->sh_qkv, &H->sh_o, &H->sh_gu, &H->sh_d, &H->sh_head};
  const int dims[5][2] = {{3 * d, d}, {d, d}, {2 * f, d}, {d, f}, {V, d}};
  int tab_ints = 0;
  for (int k = 0; k < 5; ++k)
    tab_ints += (gemm_table_ints(dims[k][0], dims[k][1], H->f32, C, gc) + 3) / 4 * 4;
  H->gemm_tab = cv.take<int>(tab_ints);
  size_t part_floats = 0;
  for (int k = 0; k < 5; ++k) {
    gemm_plan(dims[k][0], dims[k][1], H->f32, C, gc, shapes[k], nullptr, nullptr);
    part_floats = std::max(part_floats, gemm_part_bytes(*shapes[k], C) / sizeof(float));
  }
  H->part = cv.take<float>(part_floats);
  H->h = cv.take<float>((size_t)C * d);
  H->hc = cv.take<float>((size_t)C * d);
  H->q = cv.take<float>((size_t)C * d);
  H->attn_part = cv.take<float>((size_t)C * m.n_heads * H->max_splits * (m.head_dim + 2));
  H->attn_cnt = cv.take<int>((size_t)C * m.n_heads);
  H->ssq_tiles = (d + 127) / 128;
  H->ssq = cv.take<float>((size_t)H->ssq_tiles * C);
  H->cnt_o = cv.take<unsigned long long>(H->ssq_tiles);
  H->cnt_d = cv.take<unsigned long long>(H->ssq_tiles);
  H->cnt_gu = cv.take<unsigned long long>(f / 128);
  H->need_o = cv.take<int>(H->ssq_tiles);
  H->need_d = cv.take<int>(H->ssq_tiles);
  H->need_gu = cv.take<int>(f / 128);
  const int planes_x = H->f32 ? 2 : 1;  // fp32: hi and lo tf32 planes
  H->Xd = cv.take<char>((size_t)planes_x * C * d * esz);
  H->Xo = cv.take<char>((size_t)planes_x * C * d * esz);
  H->Xf = cv.take<char>((size_t)planes_x * C * f * esz);
  H->lo_d = H->f32 ? (size_t)C * d : 0;
  H->lo_f = H->f32 ? (size_t)C * f : 0;
  if (H->f32) {
    const int nl = m.n_prelude + m.n_core + m.n_coda;
    H->wsplit_elems = (size_t)nl * (4 * (size_t)d * d + 3 * (size_t)d * f) + (size_t)V * d;
    H->wsplit = cv.take<float>(2 * H->wsplit_elems);
  }
  D.logits = cv.take<float>((size_t)C * V);
  D.P = cv.take<float>((size_t)C * V);
  D.q1 = cv.take<float>((size_t)C * V);
  D.q2 = cv.take<float>((size_t)C * V);
  D.cb_val = cv.take<float>((size_t)C * ro_chunks(V));
  D.cb_idx = cv.take<int>((size_t)C * ro_chunks(V));
  D.rho = cv.take<float>((size_t)C * V);  // per row: rows of a copied chain verify in one step
  D.rho2 = cv.take<float>((size_t)C * V);
  H->rope = cv.take<float2>((size_t)H->max_pos * (m.head_dim / 2));
  H->kv = cv.take<char>((size_t)H->planes * H->S * 2 * d * esz);
  return cv.off + 256;
}

static void plan(Handle* H) {
  const lt_model_config& m = H->m;
  const lt_decode_config& dc = H->dc;
  H->f32 = m.dtype == LT_F32;
  H->mode = H->f32 ? 2 : 0;
  H->C = dc.max_branches;
  H->S = dc.max_ctx + H->C + 8;
  H->max_pos = dc.max_ctx + H->C + 8;
  H->max_splits = (H->max_pos + ATT_CH - 1) / ATT_CH;
  int n = 0;
  for (int r : {dc.d1, dc.d2, m.R})
    if (r > 0) {
      bool dup = false;
      for (int k = 0; k < n; ++k) dup |= H->tags[k] == r;
      if (!dup) H->tags[n++] = r;
    }
  std::sort(H->tags, H->tags + n);
  H->n_tags = n;
  H->plane_base.clear();
  int planes = 0;
  for (int l = 0; l < m.n_prelude; ++l) H->plane_base.push_back(planes), planes += 1;
  for (int l = 0; l < m.n_core; ++l) H->plane_base.push_back(planes), planes += m.R;
  for (int l = 0; l < m.n_coda; ++l) H->plane_base.push_back(planes), planes += n;
  H->planes = planes;
  Dev& D = H->D;
  D.d = m.d_model;
  D.V = m.vocab;
  D.R = m.R;
  D.C = H->C;
  D.S = H->S;
  D.d1 = dc.d1;
  D.d2 = dc.d2;
  D.greedy = dc.temperature == 0.f;
  D.second_mode = dc.second_mode;
  D.trace_cap = dc.trace_steps;
  D.max_ctx = dc.max_ctx;
  D.T = dc.temperature;
  D.top_p = dc.top_p;
  D.seed = dc.seed;
  D.copy_k = dc.copy_k;
  D.copy_max = dc.copy_max_len;
  D.copy_cap = dc.copy_match_cap;
  D.copy_reserve = dc.copy_reserve;
  D.copy_slack = dc.d1 > 0 ? (m.R + dc.d1 - 1) / dc.d1 : 0;
  D.copy_tau = dc.copy_tau;
  for (int r = 0; r <= 32; ++r) D.tag_of_depth[r] = -1;
  for (int k = 0; k < n; ++k) D.tag_of_depth[H->tags[k]] = k;
}

// ---------------------------------------------------------------------------
// the batched pass
// ---------------------------------------------------------------------------
#define LT_CK(x)                                   \
  do {                                             \
    cudaError_t e_ = (x);                          \
    if (e_ != cudaSuccess) return e_;              \
  } while (0)

template <typename T>
static cudaError_t gemm(Handle* H, const GemmOperand& tw, const GemmOperand& twl,
                        const GemmOperand& tx, const GemmOperand& txl, const GemmShape& s,
                        const int* flag, const GemmEpi* epi = nullptr,
                        const GemmOperand* next_w = nullptr, const GemmShape* next_s = nullptr) {
  const double esz = H->f32 ? 4.0 : 2.0, split = H->mode == 2 ? 2.0 : 1.0;
  // algorithmic bytes: the weight matrix (both tf32 halves when split), the
  // activation rows and the fp32 result rows
  const double bytes = split * esz * ((double)s.n_out * s.k + (double)H->C * s.k) +
                       4.0 * H->C * s.n_out;
  const Ctl* ctl = H->D.ctl;
  const int gate = flag == &ctl->flag_run ? 1 : flag == &ctl->flag_new ? 2 : flag == &ctl->flag_ro ? 3 : 0;
  ProfScope ps(H, H->prof_cat, bytes, gate);
  if (H->counting) H->kernels_per_step++;
  return gemm_launch(tw, twl, tx, txl, H->part, s, H->C, H->mode, flag, &H->D.ctl->err,
                     H->stream, H->use_pdl, epi, next_w, next_s);
}

// Arguments of the attention work items of layer gl (see AttnArgs).
static AttnArgs attn_args(Handle* H, int gl, const int* tagsrc, int tag_off, void* Xo) {
  Dev& D = H->D;
  AttnArgs a = {};
  a.q = (const float*)H->q;
  a.kv = H->kv;
  a.plane_base = H->plane_base[gl];
  a.tagsrc = tagsrc;
  a.tag_off = tag_off;
  a.S = H->S;
  a.d = H->m.d_model;
  a.H = H->m.n_heads;
  a.r_pos = (const int*)D.r_pos;
  a.r_blen = (const int*)D.r_blen;
  a.r_boff = (const int*)D.r_boff;
  a.lists = H->lists_override ? H->lists_override : (const int*)D.lists;
  a.chain = (const int*)D.b_chain;
  a.W = (int)WIN;
  a.max_splits = H->max_splits;
  a.opart = H->attn_part;
  a.counters = H->attn_cnt;
  a.X = Xo;
  a.lo = H->lo_d;
  a.part = (const float*)H->part;
  a.qs_shape = H->sh_qkv;
  a.C = H->C;
  a.r_slot = (const int*)D.r_slot;
  a.rope = (const float2*)H->rope;
  a.ssq = (const float*)H->ssq;
  a.ssq_tiles = H->ssq_tiles;
  a.eps = H->m.rms_eps;
  a.err = &D.ctl->err;
  return a;
}

// One resident wave of attention blocks, each streaming a contiguous range of
// (head, row, split) units (k_attn).  The shared-memory attribute is set per
// device (function attributes belong to a context), and the occupancy that
// follows from it is cached with it.
template <typename T, int HD, int NS>
static cudaError_t attention_ns(Handle* H, int gl, const int* tagsrc, int tag_off, const int* mask,
                                T* Xo, bool fused) {
  auto kern = fused ? k_attn<T, HD, NS, true> : k_attn<T, HD, NS, false>;
  const size_t smem = attn_smem_bytes<T, HD, NS>();
  static int per_sm[kMaxDev][2] = {};
  int& nb = per_sm[cur_dev()][fused ? 1 : 0];
  if (nb == 0) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return cudaErrorInvalidValue;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, 128, smem) != cudaSuccess || nb < 1)
      nb = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nb * sm_count());
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = H->stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = H->use_pdl ? 1 : 0;
  if (H->counting) H->kernels_per_step++;
  return cudaLaunchKernelEx(&cfg, kern, attn_args(H, gl, tagsrc, tag_off, (void*)Xo), mask);
}

template <typename T, int HD>
static cudaError_t attention(Handle* H, int gl, const int* tagsrc, int tag_off, const int* mask,
                             T* Xo, bool fused) {
  ProfScope ps(H, 2, 0.0);
  return attention_ns<T, HD, attn_stages<T, HD>()>(H, gl, tagsrc, tag_off, mask, Xo, fused);
}

// kind: 0 prelude (one cache), 1 shared block (cache of the row's depth), 2 coda
// (cache of the row's readout depth).
// fused: decode pass (the QKV epilogue runs inside attention, see k_attn).
template <typename T>
static cudaError_t run_layers(Handle* H, int gl0, int n, int kind, const int* mask, float* hbuf,
                              float scale, const int* flag, bool fused) {
  Dev& D = H->D;
  const lt_model_config& m = H->m;
  const int C = H->C, d = m.d_model;
  const int* tagsrc = kind == 0 ? nullptr : kind == 1 ? D.r_depth : D.r_ro;
  const int tag_off = kind == 1 ? -1 : 0;
  T* Xd = (T*)H->Xd;
  T* Xo = (T*)H->Xo;
  GemmEpi eo = {}, egu = {}, ed = {};
  eo.kind = ed.kind = EPI_RESID;
  eo.counters = H->cnt_o;
  eo.need = H->need_o;
  ed.counters = H->cnt_d;
  ed.need = H->need_d;
  eo.mask = ed.mask = egu.mask = mask;
  eo.h = ed.h = hbuf;
  eo.scale = ed.scale = scale;
  eo.X = ed.X = H->Xd;
  eo.lo = ed.lo = H->lo_d;
  eo.ssq_out = ed.ssq_out = H->ssq;
  eo.d = ed.d = egu.d = d;
  egu.kind = EPI_SWIGLU;
  egu.counters = H->cnt_gu;
  egu.need = H->need_gu;
  egu.ssq_in = H->ssq;
  egu.ssq_tiles = H->ssq_tiles;
  egu.eps = m.rms_eps;
  egu.ffn = egu.d = m.ffn;
  egu.d = d;
  egu.X = H->Xf;
  egu.lo = H->lo_f;
  for (int l = 0; l < n; ++l) {
    const int gl = gl0 + l;
    const LayerW& L = H->layers[gl];
    if (l == 0)
      LT_CK(launch(H->use_pdl, k_stage_norm<T>, dim3(C), dim3(EPI_THREADS), H->stream,
                   (const float*)hbuf, mask, (const T*)L.g1, d, C, Xd, H->lo_d, H->ssq));
    // each GEMM requests the next GEMM's weights into L2 (see k_gemm)
    LT_CK(gemm<T>(H, L.tm_qkv, L.tm_qkv_lo, H->tm_Xd, H->tm_Xd_lo, H->sh_qkv, flag, nullptr,
                  &L.tm_o, &H->sh_o));
    if (!fused)
      LT_CK(launch(H->use_pdl, k_qkv_epi<T>, dim3(C), dim3(EPI_THREADS), H->stream,
                   (const float*)H->part, H->sh_qkv, C, mask, (const int*)D.r_pos,
                   (const int*)D.r_slot, tagsrc, tag_off, H->plane_base[gl], H->S, d, m.head_dim,
                   (const float2*)H->rope, (T*)H->kv, H->q, (const float*)H->ssq, H->ssq_tiles,
                   m.rms_eps, &D.ctl->err));
    switch (m.head_dim) {
      case 32: LT_CK((attention<T, 32>(H, gl, tagsrc, tag_off, mask, Xo, fused))); break;
      case 64: LT_CK((attention<T, 64>(H, gl, tagsrc, tag_off, mask, Xo, fused))); break;
      case 96: LT_CK((attention<T, 96>(H, gl, tagsrc, tag_off, mask, Xo, fused))); break;
      default: LT_CK((attention<T, 128>(H, gl, tagsrc, tag_off, mask, Xo, fused))); break;
    }
    eo.g = L.g2;  // O: h += s * o W_o^T; X = g2 (.) h for the gate/up GEMM
    LT_CK(gemm<T>(H, L.tm_o, L.tm_o_lo, H->tm_Xo, H->tm_Xo_lo, H->sh_o, flag, &eo, &L.tm_gu,
                  &H->sh_gu));
    LT_CK(gemm<T>(H, L.tm_gu, L.tm_gu_lo, H->tm_Xd, H->tm_Xd_lo, H->sh_gu, flag, &egu, &L.tm_d,
                  &H->sh_d));
    ed.g = (l + 1 < n) ? H->layers[gl + 1].g1 : nullptr;  // next layer's g1 (.) h
    const GemmOperand* nw = (l + 1 < n) ? &H->layers[gl + 1].tm_qkv : (fused ? &H->tm_head : nullptr);
    const GemmShape* ns = (l + 1 < n) ? &H->sh_qkv : (fused ? &H->sh_head : nullptr);
    LT_CK(gemm<T>(H, L.tm_d, L.tm_d_lo, H->tm_Xf, H->tm_Xf_lo, H->sh_d, flag, &ed, nw, ns));
  }
  return cudaSuccess;
}

// Readout C of the rows in D.m_ro: coda layers on a copy of the state, final
// norm, LM head, processing.
template <typename T>
static cudaError_t run_readout(Handle* H, const int* flag, bool fused) {
  Dev& D = H->D;
  const lt_model_config& m = H->m;
  const int C = H->C, d = m.d_model;
  float* src = H->h;
  if (m.n_coda > 0) {
    LT_CK(launch(H->use_pdl, k_copy_rows<T>, dim3(C), dim3(EPI_THREADS), H->stream,
                 (const float*)H->h, (const int*)D.m_ro, d, H->hc));
    LT_CK(run_layers<T>(H, m.n_prelude + m.n_core, m.n_coda, 2, D.m_ro, H->hc, 1.f, flag, fused));
    src = H->hc;
  }
  LT_CK(launch(H->use_pdl, k_stage_norm<T>, dim3(C), dim3(EPI_THREADS), H->stream,
               (const float*)src, (const int*)D.m_ro, (const T*)H->final_norm, d, C, (T*)H->Xd,
               H->lo_d, H->ssq));
  LT_CK(gemm<T>(H, H->tm_head, H->tm_head_lo, H->tm_Xd, H->tm_Xd_lo, H->sh_head, flag));
  LT_CK(launch(H->use_pdl, k_logits, dim3(ro_chunks(m.vocab), C), dim3(RO_THREADS), H->stream,
               (const float*)H->part, H->sh_head, C, (const int*)D.m_ro, m.vocab, D.logits,
               D.cb_val, D.cb_idx, (const float*)H->ssq, H->ssq_tiles, d, m.rms_eps));
  if (D.greedy || m.vocab > RO_CL_MAXV)
    return launch(H->use_pdl, k_readout, dim3(C), dim3(1024), H->stream, (const int*)D.m_ro,
                  m.vocab, D.greedy, D.T, D.top_p, D.logits, D.P, D.ro_arg,
                  (const float*)D.cb_val, (const int*)D.cb_idx, &D.ctl->err);
  // sampled readouts: one cluster of RO_CL CTAs per row
  if (g_launch_counter) ++*g_launch_counter;
  return launch_cluster(H, k_readout_cl, dim3(RO_CL, C), (const int*)D.m_ro, m.vocab, D.T,
                        D.top_p, (const float*)D.logits, D.P, D.ro_arg, (const float*)D.cb_val,
                        (const int*)D.cb_idx, &D.ctl->err);
}

template <typename T>
static cudaError_t decode_step(Handle* H) {
  Dev& D = H->D;
  const lt_model_config& m = H->m;
  const int C = H->C;
  Ctl* ctl = D.ctl;
  LT_CK(launch(H->use_pdl, k_embed<T>, dim3(C), dim3(EPI_THREADS), H->stream, (const T*)H->embed,
               (const int*)D.r_tok, (const int*)D.m_new, m.d_model, m.vocab, H->h, &ctl->err));
  // With copy proposals a chain's rows share a depth and attend to each
  // other's cache rows of the same pass, so every row's K/V is written by the
  // QKV epilogue kernel before attention runs (the fused attention writes a
  // row's own K/V inside its own work item).
  const bool fused = D.copy_k == 0;
  H->prof_cat = 1;
  if (m.n_prelude > 0)
    LT_CK(run_layers<T>(H, 0, m.n_prelude, 0, D.m_new, H->h, 1.f, &ctl->flag_new, fused));
  H->prof_cat = 0;
  LT_CK(run_layers<T>(H, m.n_prelude, m.n_core, 1, D.m_alive, H->h, m.resid_scale,
                      &ctl->flag_run, fused));
  H->prof_cat = 1;
  LT_CK(run_readout<T>(H, &ctl->flag_ro, fused));
  if (D.greedy) {
    LT_CK(launch(H->use_pdl, k_decide, dim3(C), dim3(1024), H->stream, D));
  } else {
    // sampled decisions: one cluster of RO_CL CTAs per row
    if (g_launch_counter) ++*g_launch_counter;
    LT_CK(launch_cluster(H, k_decide_cl, dim3(RO_CL, C), D));
  }
  return launch(H->use_pdl, k_book, dim3(1), dim3(256), H->stream, D, 0, 0);
}

static cudaError_t step_once(Handle* H) {
  return H->f32 ? decode_step<float>(H) : decode_step<__nv_bfloat16>(H);
}

__global__ void k_begin(Ctl* c, int n, int ar) {
  pdl_wait();
  pdl_trigger();
  c->target_len = c->L + n;
  c->pos_limit = c->L + n - 1;
  c->finished = n <= 0;
  c->ar_mode = ar;
  c->n_commit = 0;
  c->steps = c->rows_sum = c->rows_max = 0;
  c->n_first = c->n_second = c->n_fallback = 0;
  c->gate_checks = c->gate_opens = c->branches_created = c->resid_fallback = 0;
}

__global__ void k_iota(int* a, int n) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n; k += gridDim.x * blockDim.x) a[k] = k;
}

}  // namespace lt

using namespace lt;

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------
struct lt_handle {
  Handle h;
};

static int fail(lt_handle* hd, int code, const std::string& msg) {
  if (hd) hd->h.err = msg;
  return code;
}
static int cuda_fail(lt_handle* hd, cudaError_t e, const char* where) {
  return fail(hd, LT_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

extern "C" int lt_workspace_bytes(const lt_model_config* m, const lt_decode_config* dc,
                                  size_t* out) {
  if (!out) return LT_ERR_ARG;
  int v = validate(m, dc, nullptr);
  if (v) return v;
  Handle tmp;
  tmp.m = *m;
  tmp.dc = *dc;
  plan(&tmp);
  *out = carve(&tmp, nullptr);
  return LT_OK;
}

extern "C" int lt_create(const lt_model_config* m, const lt_decode_config* dc, void* d_workspace,
                         size_t bytes, void* stream, lt_handle** out) {
  if (!out || !d_workspace) return LT_ERR_ARG;
  *out = nullptr;
  std::string why;
  int v = validate(m, dc, &why);
  if (v) return v;
  lt_handle* hd = new lt_handle();
  Handle* H = &hd->h;
  H->m = *m;
  H->dc = *dc;
  plan(H);
  const size_t need = carve(H, nullptr);
  if (bytes < need) {
    delete hd;
    return LT_ERR_CAPACITY;
  }
  char* base = (char*)(((uintptr_t)d_workspace + 255) & ~(uintptr_t)255);
  H->ws = base;
  H->ws_bytes = bytes;
  carve(H, base);
  H->stream = (cudaStream_t)stream;
  const char* e1 = getenv("LT_NO_PDL");
  const char* e2 = getenv("LT_NO_GRAPH");
  H->use_pdl = !(e1 && e1[0] == '1');
  H->use_graph = !(e2 && e2[0] == '1');
  // reducer tables of the five GEMM shapes
  const int gc = sm_count();
  const int d = m->d_model, f = m->ffn, V = m->vocab;
  GemmShape* shapes[] = {&H->sh_qkv, &H->sh_o, &H->sh_gu, &H->sh_d, &H->sh_head};
  const int dims[5][2] = {{3 * d, d}, {d, d}, {2 * f, d}, {d, f}, {V, d}};
  std::vector<int> tab;
  std::vector<int> offs;
  for (int k = 0; k < 5; ++k) {
    const int n = (gemm_table_ints(dims[k][0], dims[k][1], H->f32, H->C, gc) + 3) / 4 * 4;
    std::vector<int> t(n, 0);
    gemm_plan(dims[k][0], dims[k][1], H->f32, H->C, gc, shapes[k], t.data(),
              t.data() + 2 * shapes[k]->tiles);
    offs.push_back((int)tab.size());
    tab.insert(tab.end(), t.begin(), t.end());
  }
  // a CTA of an epilogue GEMM keeps one arrival target per tile it touches
  if (H->sh_o.jmax > GEMM_MAX_SEGS || H->sh_gu.jmax > GEMM_MAX_SEGS ||
      H->sh_d.jmax > GEMM_MAX_SEGS) {
    delete hd;
    return LT_ERR_SHAPE;
  }
  cudaError_t e = cudaMemcpy(H->gemm_tab, tab.data(), tab.size() * sizeof(int), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    delete hd;
    return LT_ERR_CUDA;
  }
  for (int k = 0; k < 5; ++k) {
    shapes[k]->tile_c = H->gemm_tab + offs[k];
    shapes[k]->cta_t0 = H->gemm_tab + offs[k] + 2 * shapes[k]->tiles;
    shapes[k]->tinfo = reinterpret_cast<const int4*>(H->gemm_tab + offs[k] + gemm_tinfo_offset(*shapes[k]));
  }
  if (H->sh_o.jmax > 8 || H->sh_gu.jmax > 8 || H->sh_d.jmax > 8) {  // epilogue table slots
    delete hd;
    return LT_ERR_SHAPE;
  }
  {  // arrivals that complete each epilogue group (O / down: per tile; gate/up: per pair)
    std::vector<int> need_o(H->ssq_tiles), need_d(H->ssq_tiles), need_gu(f / 128);
    gemm_group_need(H->sh_o, tab.data() + offs[1], 0, need_o.data());
    gemm_group_need(H->sh_gu, tab.data() + offs[2], 2, need_gu.data());
    gemm_group_need(H->sh_d, tab.data() + offs[3], 0, need_d.data());
    const size_t esz = H->f32 ? 4 : 2, px = H->f32 ? 2 : 1;
    if (cudaMemcpy(H->need_o, need_o.data(), need_o.size() * 4, cudaMemcpyHostToDevice) ||
        cudaMemcpy(H->need_d, need_d.data(), need_d.size() * 4, cudaMemcpyHostToDevice) ||
        cudaMemcpy(H->need_gu, need_gu.data(), need_gu.size() * 4, cudaMemcpyHostToDevice) ||
        cudaMemset(H->cnt_o, 0, need_o.size() * 8) || cudaMemset(H->cnt_d, 0, need_d.size() * 8) ||
        cudaMemset(H->cnt_gu, 0, need_gu.size() * 8) ||
        cudaMemset(H->Xd, 0, px * H->C * d * esz) || cudaMemset(H->Xo, 0, px * H->C * d * esz) ||
        cudaMemset(H->Xf, 0, px * H->C * f * esz) ||
        cudaMemset(H->ssq, 0, (size_t)H->ssq_tiles * H->C * 4)) {
      delete hd;
      return LT_ERR_CUDA;
    }
  }
  // activation tensor maps (B operands)
  const size_t esz = H->f32 ? 4 : 2;
  const int kc = gemm_kc(H->C, H->f32);
  if (make_operand(&H->tm_Xd, H->Xd, H->f32, H->C, d, H->C, kc) ||
      make_operand(&H->tm_Xo, H->Xo, H->f32, H->C, d, H->C, kc) ||
      make_operand(&H->tm_Xf, H->Xf, H->f32, H->C, f, H->C, kc) ||
      make_operand(&H->tm_Xd_lo, (char*)H->Xd + H->lo_d * esz, H->f32, H->C, d, H->C, kc) ||
      make_operand(&H->tm_Xo_lo, (char*)H->Xo + H->lo_d * esz, H->f32, H->C, d, H->C, kc) ||
      make_operand(&H->tm_Xf_lo, (char*)H->Xf + H->lo_f * esz, H->f32, H->C, f, H->C, kc)) {
    delete hd;
    return LT_ERR_SHAPE;
  }
  // the control block (error word, counters) starts zeroed: calls that run
  // before the first prefill (lt_block_pass) read its error word
  if (cudaMemsetAsync(H->D.ctl, 0, sizeof(Ctl), H->stream) != cudaSuccess ||
      cudaMemsetAsync(H->attn_cnt, 0, (size_t)H->C * m->n_heads * 4, H->stream) != cudaSuccess) {
    delete hd;
    return LT_ERR_CUDA;
  }
  const int half = m->head_dim / 2;
  k_rope_table<<<(H->max_pos * half + 255) / 256, 256, 0, H->stream>>>(H->rope, H->max_pos,
                                                                        m->head_dim, m->rope_theta);
  if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(H->stream) != cudaSuccess) {
    delete hd;
    return LT_ERR_CUDA;
  }
  *out = hd;
  return LT_OK;
}

extern "C" int lt_load_weights(lt_handle* hd, const void* d_embed, const void* d_final_norm,
                               const void* d_head, const void* const* d_layers) {
  if (!hd || !d_embed || !d_final_norm || !d_head || !d_layers) return LT_ERR_ARG;
  Handle* H = &hd->h;
  const lt_model_config& m = H->m;
  const int nl = m.n_prelude + m.n_core + m.n_coda, d = m.d_model, f = m.ffn;
  H->layers.assign(nl, LayerW());
  size_t wofs = 0;
  // A weight matrix's tensor maps: bf16 -> the caller's tensor; fp32 -> hi / lo
  // tf32 copies in the workspace (split once here, at load time).
  const int kc = gemm_kc(H->C, H->f32);
  auto maps = [&](const void* w, int rows, int k, GemmOperand* hi, GemmOperand* lo) -> int {
    if (!H->f32) {
      if (make_operand(hi, w, false, rows, k, GEMM_BM, kc)) return -1;
      *lo = *hi;
      return 0;
    }
    const size_t n = (size_t)rows * k;
    float* wh = H->wsplit + wofs;
    float* wl = H->wsplit + H->wsplit_elems + wofs;
    wofs += n;
    if (wofs > H->wsplit_elems) return -2;
    if (split_tf32((const float*)w, wh, wl, n, H->stream) != cudaSuccess) return -3;
    if (make_operand(hi, wh, true, rows, k, GEMM_BM, kc) ||
        make_operand(lo, wl, true, rows, k, GEMM_BM, kc))
      return -1;
    return 0;
  };
  for (int l = 0; l < nl; ++l) {
    LayerW& L = H->layers[l];
    const void* const* p = d_layers + 6 * l;
    for (int k = 0; k < 6; ++k)
      if (!p[k]) return fail(hd, LT_ERR_ARG, "null layer tensor");
    L.g1 = p[0];
    L.wqkv = p[1];
    L.wo = p[2];
    L.g2 = p[3];
    L.wgu = p[4];
    L.wd = p[5];
    if (maps(L.wqkv, 3 * d, d, &L.tm_qkv, &L.tm_qkv_lo) ||
        maps(L.wo, d, d, &L.tm_o, &L.tm_o_lo) ||
        maps(L.wgu, 2 * f, d, &L.tm_gu, &L.tm_gu_lo) ||
        maps(L.wd, d, f, &L.tm_d, &L.tm_d_lo))
      return fail(hd, LT_ERR_SHAPE, "weight tensor map (alignment?)");
  }
  if (maps(d_head, m.vocab, d, &H->tm_head, &H->tm_head_lo))
    return fail(hd, LT_ERR_SHAPE, "head tensor map");
  if (cudaStreamSynchronize(H->stream) != cudaSuccess) return fail(hd, LT_ERR_CUDA, "weight split");
  H->embed = d_embed;
  H->final_norm = d_final_norm;
  H->head = d_head;
  H->loaded = true;
  if (H->graph) {
    cudaGraphExecDestroy(H->graph);
    H->graph = nullptr;
  }
  return LT_OK;
}

template <typename T>
static int prefill_t(lt_handle* hd, const int32_t* h_tokens, int n, int32_t* h_first,
                     int32_t* h_argmax, float* d_logits) {
  Handle* H = &hd->h;
  Dev& D = H->D;
  const lt_model_config& m = H->m;
  const int C = H->C;
  cudaStream_t st = H->stream;
  cudaError_t e;
  // fresh state
  Ctl c0 = {};
  c0.L = n;
  c0.next_uid = 0;
  if ((e = cudaMemcpyAsync(D.ctl, &c0, sizeof(Ctl), cudaMemcpyHostToDevice, st))) return cuda_fail(hd, e, "ctl");
  const int words = (H->S + 31) / 32;
  std::vector<unsigned int> bits(words, 0u);
  for (int s = 0; s < n; ++s) bits[s >> 5] |= 1u << (s & 31);
  std::vector<int> zeros((size_t)C * WIN, 0);
  if ((e = cudaMemcpyAsync(D.slot_bits, bits.data(), words * 4, cudaMemcpyHostToDevice, st)) ||
      (e = cudaMemcpyAsync(D.committed, h_tokens, n * 4, cudaMemcpyHostToDevice, st)) ||
      (e = cudaMemsetAsync(D.b_alive, 0, C * 4, st)) ||
      (e = cudaMemsetAsync(D.b_chain, 0, (size_t)C * WIN * 4, st)) ||
      (e = cudaMemsetAsync(H->h, 0, (size_t)C * m.d_model * 4, st)))
    return cuda_fail(hd, e, "prefill init");
  k_iota<<<32, 256, 0, st>>>(D.lists, n);
  const int dep_tags = H->n_tags;
  const int gl_core = m.n_prelude;
  for (int c0p = 0; c0p < n; c0p += C) {
    const int cnt = std::min(C, n - c0p);
    const bool last = c0p + cnt == n;
    if ((e = launch(false, k_prefill_rows, dim3(1), dim3(64), st, D, c0p, cnt, n, 0, -1))) return cuda_fail(hd, e, "rows");
    if ((e = launch(false, k_embed<T>, dim3(C), dim3(EPI_THREADS), st, (const T*)H->embed,
                    (const int*)D.r_tok, (const int*)D.m_new, m.d_model, m.vocab, H->h, &D.ctl->err)))
      return cuda_fail(hd, e, "embed");
    if (m.n_prelude > 0 && (e = run_layers<T>(H, 0, m.n_prelude, 0, D.m_alive, H->h, 1.f, nullptr, false)))
      return cuda_fail(hd, e, "prelude");
    for (int r = 1; r <= m.R; ++r) {
      const int tag = D.tag_of_depth[r];
      if ((e = launch(false, k_prefill_rows, dim3(1), dim3(64), st, D, c0p, cnt, n, r, tag)))
        return cuda_fail(hd, e, "rows");
      if ((e = run_layers<T>(H, gl_core, m.n_core, 1, D.m_alive, H->h, m.resid_scale, nullptr, false)))
        return cuda_fail(hd, e, "core");
      if (tag < 0) continue;
      const bool need_head = (last && r == m.R) || h_argmax || d_logits;
      if (need_head) {
        if ((e = run_readout<T>(H, nullptr, false))) return cuda_fail(hd, e, "readout");
        if (d_logits)
          for (int k = 0; k < cnt; ++k)
            if ((e = cudaMemcpyAsync(d_logits + ((size_t)(c0p + k) * dep_tags + tag) * m.vocab,
                                     D.logits + (size_t)k * m.vocab, m.vocab * 4,
                                     cudaMemcpyDeviceToDevice, st)))
              return cuda_fail(hd, e, "logits copy");
        if (h_argmax) {
          std::vector<int> a(cnt);
          if ((e = cudaMemcpyAsync(a.data(), D.ro_arg, cnt * 4, cudaMemcpyDeviceToHost, st)) ||
              (e = cudaStreamSynchronize(st)))
            return cuda_fail(hd, e, "argmax copy");
          for (int k = 0; k < cnt; ++k) h_argmax[(size_t)(c0p + k) * dep_tags + tag] = a[k];
        }
      } else if (m.n_coda > 0) {
        // coda caches of this readout depth are still needed by later positions
        if ((e = launch(false, k_copy_rows<T>, dim3(C), dim3(EPI_THREADS), st, (const float*)H->h,
                        (const int*)D.m_ro, m.d_model, H->hc)) ||
            (e = run_layers<T>(H, m.n_prelude + m.n_core, m.n_coda, 2, D.m_ro, H->hc, 1.f, nullptr, false)))
          return cuda_fail(hd, e, "coda");
      }
      if (last && r == m.R) {
        if ((e = launch(false, k_first_token, dim3(1), dim3(1024), st, D, cnt - 1, n)))
          return cuda_fail(hd, e, "first token");
      }
    }
  }
  int first = -1;
  Ctl cc;
  if ((e = cudaMemcpyAsync(&first, D.committed + n, 4, cudaMemcpyDeviceToHost, st)) ||
      (e = cudaMemcpyAsync(&cc, D.ctl, sizeof(Ctl), cudaMemcpyDeviceToHost, st)) ||
      (e = cudaStreamSynchronize(st)))
    return cuda_fail(hd, e, "prefill sync");
  if (cc.err) return fail(hd, LT_ERR_DEVICE_CHECK, "device error " + std::to_string(cc.err));
  if (h_first) *h_first = first;
  H->P = n;
  H->prefilled = true;
  H->begun = false;
  return LT_OK;
}

extern "C" int lt_prefill(lt_handle* hd, const int32_t* h_tokens, int n, int32_t* h_first,
                          int32_t* h_argmax, float* d_logits) {
  if (!hd || !h_tokens || n <= 0) return LT_ERR_ARG;
  Handle* H = &hd->h;
  if (!H->loaded) return fail(hd, LT_ERR_STATE, "weights not loaded");
  if (n + 1 > H->dc.max_ctx) return fail(hd, LT_ERR_CAPACITY, "prompt longer than max_ctx - 1");
  if (H->S > MAX_SLOT_WORDS * 32)
    return fail(hd, LT_ERR_CAPACITY, "decoding needs max_ctx + max_branches + 8 <= 65536 slots");
  for (int k = 0; k < n; ++k)
    if (h_tokens[k] < 0 || h_tokens[k] >= H->m.vocab) return fail(hd, LT_ERR_ARG, "token id out of range");
  return H->f32 ? prefill_t<float>(hd, h_tokens, n, h_first, h_argmax, d_logits)
                : prefill_t<__nv_bfloat16>(hd, h_tokens, n, h_first, h_argmax, d_logits);
}

static int read_ctl(lt_handle* hd, Ctl* c) {
  Handle* H = &hd->h;
  cudaError_t e;
  if ((e = cudaMemcpyAsync(c, H->D.ctl, sizeof(Ctl), cudaMemcpyDeviceToHost, H->stream)) ||
      (e = cudaStreamSynchronize(H->stream)))
    return cuda_fail(hd, e, "ctl readback");
  if (c->err) {
    const int code = (c->err == DEV_TABLE_FULL || c->err == DEV_SLOTS_FULL || c->err == DEV_CHAIN)
                         ? LT_ERR_CAPACITY
                         : LT_ERR_DEVICE_CHECK;
    return fail(hd, code, "device error " + std::to_string(c->err));
  }
  return LT_OK;
}

// Running totals of the device counters since the current decode began.
static void fill_stats(const Ctl& c, lt_stats* st) {
  st->steps = c.steps;
  st->rows_sum = c.rows_sum;
  st->rows_max = c.rows_max;
  st->n_first = c.n_first;
  st->n_second = c.n_second;
  st->n_fallback = c.n_fallback;
  st->gate_checks = c.gate_checks;
  st->gate_opens = c.gate_opens;
  st->branches_created = c.branches_created;
  st->resid_fallback = c.resid_fallback;
  st->committed_len = c.L;
  st->copy_chains = c.copy_chains;
  st->copy_rows = c.copy_rows;
  st->copy_cut = c.copy_cut;
  st->n_copy = c.n_copy;
}

static int ensure_graph(lt_handle* hd) {
  Handle* H = &hd->h;
  if (!H->use_graph || H->graph) return LT_OK;
  cudaGraph_t g = nullptr;
  cudaError_t e = cudaStreamBeginCapture(H->stream, cudaStreamCaptureModeThreadLocal);
  if (e) return cuda_fail(hd, e, "begin capture");
  H->kernels_per_step = 0;
  int other = 0;
  g_launch_counter = &other;
  H->counting = true;
  cudaError_t e2 = step_once(H);
  H->counting = false;
  g_launch_counter = nullptr;
  H->kernels_per_step += other;
  e = cudaStreamEndCapture(H->stream, &g);
  if (e2) return cuda_fail(hd, e2, "capture step");
  if (e) return cuda_fail(hd, e, "end capture");
  e = cudaGraphInstantiate(&H->graph, g, 0);
  cudaGraphDestroy(g);
  if (e) {
    H->graph = nullptr;
    return cuda_fail(hd, e, "instantiate");
  }
  return LT_OK;
}

static int run_steps(lt_handle* hd, int k) {
  Handle* H = &hd->h;
  for (int s = 0; s < k; ++s) {
    cudaError_t e = H->graph ? cudaGraphLaunch(H->graph, H->stream) : step_once(H);
    if (e) return cuda_fail(hd, e, "step launch");
  }
  return LT_OK;
}

static int begin(lt_handle* hd, int n, int ar) {
  Handle* H = &hd->h;
  cudaError_t e;
  if ((e = launch(false, k_begin, dim3(1), dim3(1), H->stream, H->D.ctl, n, ar)) ||
      (e = launch(false, k_book, dim3(1), dim3(256), H->stream, H->D, 1, 0)))
    return cuda_fail(hd, e, "begin");
  H->begun = true;
  return LT_OK;
}

extern "C" int lt_generate(lt_handle* hd, int ar_mode, int n, int32_t* h_out, lt_stats* st) {
  if (!hd || n < 0) return LT_ERR_ARG;
  Handle* H = &hd->h;
  if (!H->prefilled) return fail(hd, LT_ERR_STATE, "prefill first");
  Ctl c;
  int rc = read_ctl(hd, &c);
  if (rc) return rc;
  const int L0 = c.L;
  if (L0 + n > H->dc.max_ctx) return fail(hd, LT_ERR_CAPACITY, "max_ctx exceeded");
  if ((rc = begin(hd, n, ar_mode ? 1 : 0))) return rc;
  if ((rc = ensure_graph(hd))) return rc;
  int remaining = n;
  while (remaining > 0) {
    // a step commits at least 0 tokens and the device stops at the target, so
    // `remaining` steps cannot overshoot (copied chains can commit several)
    if ((rc = run_steps(hd, remaining))) return rc;
    if ((rc = read_ctl(hd, &c))) return rc;
    remaining = L0 + n - c.L;
    if (c.finished && remaining > 0) return fail(hd, LT_ERR_DEVICE_CHECK, "stopped early");
  }
  cudaError_t e;
  if (h_out && n > 0) {
    if ((e = cudaMemcpyAsync(h_out, H->D.committed + L0, n * 4, cudaMemcpyDeviceToHost, H->stream)) ||
        (e = cudaStreamSynchronize(H->stream)))
      return cuda_fail(hd, e, "tokens readback");
  }
  if (st) fill_stats(c, st);
  H->begun = false;
  return LT_OK;
}

extern "C" int lt_get_stats(lt_handle* hd, lt_stats* st) {
  if (!hd || !st) return LT_ERR_ARG;
  Handle* H = &hd->h;
  if (!H->prefilled) return fail(hd, LT_ERR_STATE, "prefill first");
  Ctl c;
  const int rc = read_ctl(hd, &c);
  if (rc) return rc;
  fill_stats(c, st);
  return LT_OK;
}

extern "C" int lt_decode_step(lt_handle* hd, int ar_mode, int32_t* h_tok, int* n_committed,
                              lt_step_info* info) {
  if (!hd) return LT_ERR_ARG;
  Handle* H = &hd->h;
  if (!H->prefilled) return fail(hd, LT_ERR_STATE, "prefill first");
  int rc;
  Ctl c;
  if (!H->begun) {
    if ((rc = read_ctl(hd, &c))) return rc;
    const int room = H->dc.max_ctx - c.L;
    if ((rc = begin(hd, std::min(H->dc.max_new, room), ar_mode ? 1 : 0))) return rc;
  }
  if ((rc = read_ctl(hd, &c))) return rc;
  const Ctl c0 = c;
  const int before = c.n_commit;
  if ((rc = ensure_graph(hd))) return rc;
  if ((rc = run_steps(hd, 1))) return rc;
  if ((rc = read_ctl(hd, &c))) return rc;
  const int got = c.n_commit - before;
  if (info) {  // this pass's share of the running counters
    info->step = c.steps;
    info->rows = c.rows_sum - c0.rows_sum;
    info->n_committed = got;
    info->n_first = c.n_first - c0.n_first;
    info->n_second = c.n_second - c0.n_second;
    info->n_fallback = c.n_fallback - c0.n_fallback;
    info->n_copy = c.n_copy - c0.n_copy;
    info->gate_checks = c.gate_checks - c0.gate_checks;
    info->gate_opens = c.gate_opens - c0.gate_opens;
    info->branches_created = c.branches_created - c0.branches_created;
    info->committed_len = c.L;
    info->finished = c.finished;
  }
  if (got > 0 && h_tok) {
    cudaError_t e;
    if ((e = cudaMemcpyAsync(h_tok, H->D.log_tok + c.n_commit - 1, 4, cudaMemcpyDeviceToHost, H->stream)) ||
        (e = cudaStreamSynchronize(H->stream)))
      return cuda_fail(hd, e, "log readback");
  }
  if (n_committed) *n_committed = got;
  if (c.finished) H->begun = false;
  return LT_OK;
}

extern "C" int lt_read_log(lt_handle* hd, int32_t* h_tok, int32_t* h_src, int32_t* h_step, int n) {
  if (!hd || n < 0) return LT_ERR_ARG;
  Handle* H = &hd->h;
  cudaError_t e;
  if ((h_tok && (e = cudaMemcpyAsync(h_tok, H->D.log_tok, n * 4, cudaMemcpyDeviceToHost, H->stream))) ||
      (h_src && (e = cudaMemcpyAsync(h_src, H->D.log_src, n * 4, cudaMemcpyDeviceToHost, H->stream))) ||
      (h_step && (e = cudaMemcpyAsync(h_step, H->D.log_step, n * 4, cudaMemcpyDeviceToHost, H->stream))) ||
      (e = cudaStreamSynchronize(H->stream)))
    return cuda_fail(hd, e, "log");
  return LT_OK;
}

extern "C" int lt_read_trace(lt_handle* hd, int32_t* h_trace, int n_steps) {
  if (!hd || !h_trace || n_steps < 0) return LT_ERR_ARG;
  Handle* H = &hd->h;
  if (n_steps > H->dc.trace_steps) return fail(hd, LT_ERR_CAPACITY, "trace_steps too small");
  cudaError_t e;
  if ((e = cudaMemcpyAsync(h_trace, H->D.trace, (size_t)n_steps * H->C * 16, cudaMemcpyDeviceToHost, H->stream)) ||
      (e = cudaStreamSynchronize(H->stream)))
    return cuda_fail(hd, e, "trace");
  return LT_OK;
}

extern "C" int lt_read_committed(lt_handle* hd, int32_t* h_tokens, int32_t* h_slots, int* h_len) {
  if (!hd) return LT_ERR_ARG;
  Handle* H = &hd->h;
  Ctl c;
  int rc = read_ctl(hd, &c);
  if (rc) return rc;
  cudaError_t e;
  if ((h_tokens && (e = cudaMemcpyAsync(h_tokens, H->D.committed, c.L * 4, cudaMemcpyDeviceToHost, H->stream))) ||
      (h_slots && (e = cudaMemcpyAsync(h_slots, H->D.lists, c.L * 4, cudaMemcpyDeviceToHost, H->stream))) ||
      (e = cudaStreamSynchronize(H->stream)))
    return cuda_fail(hd, e, "committed");
  if (h_len) *h_len = c.L;
  return LT_OK;
}

extern "C" int lt_read_branch_table(lt_handle* hd, int32_t* h_table) {
  if (!hd || !h_table) return LT_ERR_ARG;
  Handle* H = &hd->h;
  Dev& D = H->D;
  int* cols[] = {D.b_alive, D.b_uid, D.b_parent, D.b_slot, D.b_pos, D.b_tok, D.b_depth,
                 D.b_x1, D.b_x2, D.b_gate, D.b_c1, D.b_c2};
  cudaError_t e = cudaSuccess;
  for (int k = 0; k < 12 && !e; ++k)
    e = cudaMemcpyAsync(h_table + k * H->C, cols[k], H->C * 4, cudaMemcpyDeviceToHost, H->stream);
  if (e || (e = cudaStreamSynchronize(H->stream))) return cuda_fail(hd, e, "table");
  return LT_OK;
}

extern "C" int lt_read_readouts(lt_handle* hd, float* h_logits, float* h_probs, int32_t* h_arg,
                                int32_t* h_rows) {
  if (!hd) return LT_ERR_ARG;
  Handle* H = &hd->h;
  Dev& D = H->D;
  const size_t n = (size_t)H->C * H->m.vocab;
  cudaError_t e;
  if ((h_logits && (e = cudaMemcpyAsync(h_logits, D.logits, n * 4, cudaMemcpyDeviceToHost, H->stream))) ||
      (h_probs && (e = cudaMemcpyAsync(h_probs, D.P, n * 4, cudaMemcpyDeviceToHost, H->stream))) ||
      (h_arg && (e = cudaMemcpyAsync(h_arg, D.ro_arg, H->C * 4, cudaMemcpyDeviceToHost, H->stream))) ||
      (e = cudaStreamSynchronize(H->stream)))
    return cuda_fail(hd, e, "readouts");
  (void)h_rows;
  return LT_OK;
}

extern "C" int lt_reset(lt_handle* hd) {
  if (!hd) return LT_ERR_ARG;
  hd->h.prefilled = false;
  hd->h.begun = false;
  return LT_OK;
}

extern "C" const char* lt_last_error(const lt_handle* hd) {
  return hd ? hd->h.err.c_str() : "null handle";
}

extern "C" void lt_destroy(lt_handle* hd) {
  if (!hd) return;
  if (hd->h.graph) cudaGraphExecDestroy(hd->h.graph);
  if (hd->h.pass_graph) cudaGraphExecDestroy(hd->h.pass_graph);
  delete hd;
}

extern "C" int lt_profile_steps(lt_handle* hd, int ar_mode, int n_steps, lt_profile* out) {
  if (!hd || !out || n_steps <= 0) return LT_ERR_ARG;
  Handle* H = &hd->h;
  if (!H->prefilled) return fail(hd, LT_ERR_STATE, "prefill first");
  int rc;
  Ctl c;
  if (!H->begun) {
    if ((rc = read_ctl(hd, &c))) return rc;
    const int room = H->dc.max_ctx - c.L;
    if ((rc = begin(hd, std::min(H->dc.max_new, room), ar_mode ? 1 : 0))) return rc;
  }
  memset(out, 0, sizeof(*out));
  const bool pdl = H->use_pdl;
  H->use_pdl = false;  // clean per-kernel intervals
  cudaEvent_t s0, s1;
  cudaEventCreate(&s0);
  cudaEventCreate(&s1);
  const lt_model_config& m = H->m;
  const double esz = H->f32 ? 4.0 : 2.0;
  std::vector<int> pos(H->C), on(H->C);
  for (int k = 0; k < n_steps; ++k) {
    if ((rc = read_ctl(hd, &c))) break;
    if (c.finished) break;
    cudaMemcpy(pos.data(), H->D.r_pos, H->C * 4, cudaMemcpyDeviceToHost);
    cudaMemcpy(on.data(), H->D.m_alive, H->C * 4, cudaMemcpyDeviceToHost);
    for (int i = 0; i < H->C; ++i)
      if (on[i]) {
        // per row: every shared-block layer reads pos+1 cached K and V rows and
        // writes its own (one depth plane)
        out->kv_bytes += (double)m.n_core * (pos[i] + 2) * 2.0 * m.d_model * esz;
        out->rows += 1;
      }
    H->evs.clear();
    H->profiling = true;
    cudaEventRecord(s0, H->stream);
    cudaError_t e = step_once(H);
    cudaEventRecord(s1, H->stream);
    H->profiling = false;
    if (e || (e = cudaStreamSynchronize(H->stream))) {
      rc = cuda_fail(hd, e, "profiled step");
      break;
    }
    float ms = 0.f;
    cudaEventElapsedTime(&ms, s0, s1);
    out->step_ms += ms;
    out->steps += 1;
    for (auto& ev : H->evs) {
      float t = 0.f;
      cudaEventElapsedTime(&t, ev.a, ev.b);
      // a GEMM whose flag was clear this step exited without reading its weights
      const int live = ev.gate == 0 || (ev.gate == 1 && c.flag_run) ||
                       (ev.gate == 2 && c.flag_new) || (ev.gate == 3 && c.flag_ro);
      if (!live) ev.bytes = 0.0;
      if (ev.kind == 0) {
        out->gemm_core_ms += t;
        out->gemm_core_launches += 1;
        out->gemm_core_bytes += ev.bytes;
      } else if (ev.kind == 1) {
        out->gemm_other_ms += t;
        out->gemm_other_launches += 1;
        out->gemm_other_bytes += ev.bytes;
      } else {
        out->attn_ms += t;
        out->attn_launches += 1;
      }
      cudaEventDestroy(ev.a);
      cudaEventDestroy(ev.b);
    }
    H->evs.clear();
  }
  out->weight_bytes_core = esz * (H->mode == 2 ? 2.0 : 1.0) * m.n_core *
                           (4.0 * m.d_model * m.d_model + 3.0 * m.d_model * m.ffn);
  cudaEventDestroy(s0);
  cudaEventDestroy(s1);
  H->use_pdl = pdl;
  if (!rc && (rc = read_ctl(hd, &c)) == 0 && c.finished) H->begun = false;
  return rc;
}

// The shared-block GEMMs of one decode pass alone (QKV, O + residual,
// gate/up + SwiGLU, down + residual per layer), in the step's order and launch
// configuration, over the rows of the last step.
template <typename T>
static cudaError_t run_gemms_only(Handle* H) {
  Dev& D = H->D;
  const lt_model_config& m = H->m;
  GemmEpi eo = {}, egu = {}, ed = {};
  eo.kind = ed.kind = EPI_RESID;
  eo.counters = H->cnt_o;
  eo.need = H->need_o;
  ed.counters = H->cnt_d;
  ed.need = H->need_d;
  eo.mask = ed.mask = egu.mask = D.m_alive;
  eo.h = ed.h = H->h;
  eo.scale = ed.scale = m.resid_scale;
  eo.X = ed.X = H->Xd;
  eo.lo = ed.lo = H->lo_d;
  eo.ssq_out = ed.ssq_out = H->ssq;
  eo.d = ed.d = egu.d = m.d_model;
  egu.kind = EPI_SWIGLU;
  egu.counters = H->cnt_gu;
  egu.need = H->need_gu;
  egu.ssq_in = H->ssq;
  egu.ssq_tiles = H->ssq_tiles;
  egu.eps = m.rms_eps;
  egu.ffn = m.ffn;
  egu.d = m.d_model;
  egu.X = H->Xf;
  egu.lo = H->lo_f;
  for (int l = 0; l < m.n_core; ++l) {
    const int gl = m.n_prelude + l;
    const LayerW& L = H->layers[gl];
    LT_CK(gemm<T>(H, L.tm_qkv, L.tm_qkv_lo, H->tm_Xd, H->tm_Xd_lo, H->sh_qkv, nullptr));
    eo.g = L.g2;
    LT_CK(gemm<T>(H, L.tm_o, L.tm_o_lo, H->tm_Xo, H->tm_Xo_lo, H->sh_o, nullptr, &eo));
    LT_CK(gemm<T>(H, L.tm_gu, L.tm_gu_lo, H->tm_Xd, H->tm_Xd_lo, H->sh_gu, nullptr, &egu));
    ed.g = l + 1 < m.n_core ? H->layers[gl + 1].g1 : nullptr;
    LT_CK(gemm<T>(H, L.tm_d, L.tm_d_lo, H->tm_Xf, H->tm_Xf_lo, H->sh_d, nullptr, &ed));
  }
  return cudaSuccess;
}

extern "C" int lt_profile_gemms(lt_handle* hd, int n_iters, double* h_out) {
  if (!hd || !h_out || n_iters < 1) return LT_ERR_ARG;
  Handle* H = &hd->h;
  if (!H->loaded) return fail(hd, LT_ERR_STATE, "weights not loaded");
  const lt_model_config& m = H->m;
  cudaStream_t st = H->stream;
  double bytes = 0.0;
  const double esz = H->f32 ? 4.0 : 2.0, split = H->mode == 2 ? 2.0 : 1.0;
  for (const GemmShape* s : {&H->sh_qkv, &H->sh_o, &H->sh_gu, &H->sh_d})
    bytes += split * esz * ((double)s->n_out * s->k + (double)H->C * s->k) + 4.0 * H->C * s->n_out;
  bytes *= m.n_core;
  cudaGraph_t g = nullptr;
  cudaGraphExec_t ge = nullptr;
  cudaError_t e = cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal);
  if (e) return cuda_fail(hd, e, "capture");
  cudaError_t e2 = H->f32 ? run_gemms_only<float>(H) : run_gemms_only<__nv_bfloat16>(H);
  e = cudaStreamEndCapture(st, &g);
  if (e2 || e || (e = cudaGraphInstantiate(&ge, g, 0))) {
    if (g) cudaGraphDestroy(g);
    return cuda_fail(hd, e2 ? e2 : e, "gemm graph");
  }
  cudaGraphDestroy(g);
  cudaEvent_t a, b;
  cudaEventCreate(&a);
  cudaEventCreate(&b);
  int rc = LT_OK;
  // one untimed replay (first-touch of the graph), then the timed ones
  if ((e = cudaGraphLaunch(ge, st)) || (e = cudaEventRecord(a, st))) rc = cuda_fail(hd, e, "replay");
  for (int k = 0; k < n_iters && !rc; ++k)
    if ((e = cudaGraphLaunch(ge, st))) rc = cuda_fail(hd, e, "replay");
  float ms = 0.f;
  if (!rc && ((e = cudaEventRecord(b, st)) || (e = cudaStreamSynchronize(st)) ||
              (e = cudaEventElapsedTime(&ms, a, b))))
    rc = cuda_fail(hd, e, "replay timing");
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  cudaGraphExecDestroy(ge);
  if (rc) return rc;
  h_out[0] = ms / n_iters;
  h_out[1] = bytes;
  h_out[2] = 4.0 * m.n_core;
  // the GEMMs' epilogues overwrote the hidden states: no decode state survives
  H->prefilled = false;
  H->begun = false;
  Ctl c;
  return read_ctl(hd, &c);
}

extern "C" int lt_get_info(lt_handle* hd, lt_info* out) {
  if (!hd || !out) return LT_ERR_ARG;
  Handle* H = &hd->h;
  int rc = ensure_graph(hd);
  if (rc) return rc;
  const lt_model_config& m = H->m;
  const double esz = H->f32 ? 4.0 : 2.0;
  out->kernels_per_step = H->kernels_per_step;
  out->gemm_grid = H->sh_qkv.grid;
  out->n_tags = H->n_tags;
  out->kv_slots = H->S;
  out->workspace_bytes = (double)H->ws_bytes;
  out->weight_bytes_core = esz * m.n_core * (4.0 * m.d_model * m.d_model + 3.0 * m.d_model * m.ffn);
  const int nl = m.n_prelude + m.n_coda;
  out->weight_bytes_prelude_coda = esz * nl * (4.0 * m.d_model * m.d_model + 3.0 * m.d_model * m.ffn);
  out->weight_bytes_head = esz * (double)m.vocab * m.d_model;
  return LT_OK;
}

// Explicit edits of the branch tree between steps (see the header).
static int tree_edit(lt_handle* hd, int mode, int32_t uid) {
  if (!hd) return LT_ERR_ARG;
  Handle* H = &hd->h;
  if (!H->prefilled || !H->begun) return fail(hd, LT_ERR_STATE, "no decode in progress");
  std::vector<int> t(12 * H->C);
  int rc = lt_read_branch_table(hd, t.data());
  if (rc) return rc;
  Ctl c;
  if ((rc = read_ctl(hd, &c))) return rc;
  const int C = H->C;
  int e = -1, root = -1;
  for (int k = 0; k < C; ++k) {
    if (!t[k]) continue;
    if (t[C + k] == uid) e = k;
    if (t[4 * C + k] == c.L - 1) root = k;
  }
  if (e < 0) return fail(hd, LT_ERR_ARG, "no live branch with this uid");
  if (e == root) return fail(hd, LT_ERR_ARG, "the root cannot be edited");
  if (mode == 3 && (root < 0 || t[2 * C + e] != t[C + root]))
    return fail(hd, LT_ERR_ARG, "only a child of the root can be committed");
  if (c.finished) return fail(hd, LT_ERR_STATE, "decode finished");
  cudaError_t er = launch(false, k_book, dim3(1), dim3(256), H->stream, H->D, mode, (int)uid);
  if (er) return cuda_fail(hd, er, "tree edit");
  if ((rc = read_ctl(hd, &c))) return rc;
  if (c.finished) H->begun = false;
  return LT_OK;
}

extern "C" int lt_rollback_branch(lt_handle* hd, int32_t uid) { return tree_edit(hd, 2, uid); }
extern "C" int lt_commit_branch(lt_handle* hd, int32_t uid) { return tree_edit(hd, 3, uid); }

// ---------------------------------------------------------------------------
// one shared-block pass over caller-specified rows (kernel sweep)
// ---------------------------------------------------------------------------
__global__ void k_pass_rows(Dev D, int n, const int* __restrict__ lists) {
  pdl_wait();
  pdl_trigger();
  for (int k = threadIdx.x; k < D.C; k += blockDim.x) {
    const int on = k < n;
    const int pos = on ? D.r_pos[k] : 0;
    D.m_alive[k] = on;
    D.m_new[k] = 0;
    D.m_ro[k] = 0;
    D.r_ro[k] = -1;
    D.r_slot[k] = on ? lists[D.r_boff[k] + pos] : 0;
    D.r_blen[k] = pos + 1;
  }
}

extern "C" int lt_kv_pool(lt_handle* hd, void** d_pool, size_t* bytes, int* n_planes,
                          int* n_slots, int* plane_core0) {
  if (!hd) return LT_ERR_ARG;
  Handle* H = &hd->h;
  if (d_pool) *d_pool = H->kv;
  if (bytes) *bytes = (size_t)H->planes * H->S * 2 * H->m.d_model * (H->f32 ? 4 : 2);
  if (n_planes) *n_planes = H->planes;
  if (n_slots) *n_slots = H->S;
  if (plane_core0) *plane_core0 = H->plane_base[H->m.n_prelude];
  return LT_OK;
}

extern "C" int lt_block_pass(lt_handle* hd, int n_rows, const int32_t* h_depth,
                             const int32_t* h_pos, const int32_t* d_lists,
                             const int32_t* h_list_off, float* d_hidden, int iters,
                             float* h_ms) {
  if (!hd || !h_depth || !h_pos || !d_lists || !h_list_off || !d_hidden || iters < 1)
    return LT_ERR_ARG;
  Handle* H = &hd->h;
  if (!H->loaded) return fail(hd, LT_ERR_STATE, "weights not loaded");
  const int C = H->C, d = H->m.d_model;
  if (n_rows < 1 || n_rows > C) return fail(hd, LT_ERR_CAPACITY, "n_rows exceeds max_branches");
  std::vector<int> pos(C, 0), dep(C, 1), off(C, 0);
  for (int i = 0; i < n_rows; ++i) {
    if (h_depth[i] < 1 || h_depth[i] > H->m.R) return fail(hd, LT_ERR_ARG, "depth out of 1..R");
    if (h_pos[i] < 0 || h_pos[i] >= H->max_pos) return fail(hd, LT_ERR_ARG, "position out of range");
    if (h_list_off[i] < 0) return fail(hd, LT_ERR_ARG, "negative list offset");
    pos[i] = h_pos[i];
    dep[i] = h_depth[i];
    off[i] = h_list_off[i];
  }
  Dev& D = H->D;
  cudaStream_t st = H->stream;
  cudaError_t e;
  if ((e = cudaMemcpyAsync(D.r_pos, pos.data(), C * 4, cudaMemcpyHostToDevice, st)) ||
      (e = cudaMemcpyAsync(D.r_depth, dep.data(), C * 4, cudaMemcpyHostToDevice, st)) ||
      (e = cudaMemcpyAsync(D.r_boff, off.data(), C * 4, cudaMemcpyHostToDevice, st)) ||
      (e = launch(false, k_pass_rows, dim3(1), dim3(64), st, D, n_rows, (const int*)d_lists)) ||
      (e = cudaMemcpyAsync(H->h, d_hidden, (size_t)n_rows * d * 4, cudaMemcpyDeviceToDevice, st)))
    return cuda_fail(hd, e, "block pass setup");
  H->prefilled = false;  // the row arrays and caches no longer hold a decode state
  H->begun = false;
  H->lists_override = d_lists;
  auto pass = [&]() -> cudaError_t {
    return H->f32 ? run_layers<float>(H, H->m.n_prelude, H->m.n_core, 1, D.m_alive, H->h,
                                      H->m.resid_scale, nullptr, true)
                  : run_layers<__nv_bfloat16>(H, H->m.n_prelude, H->m.n_core, 1, D.m_alive,
                                              H->h, H->m.resid_scale, nullptr, true);
  };
  int rc = LT_OK;
  if (iters == 1 && !h_ms) {
    if ((e = pass())) rc = cuda_fail(hd, e, "block pass");
  } else {
    // one graph of the pass, replayed; events on the handle's stream around each replay
    if (H->pass_graph && H->pass_graph_rows != n_rows) {
      cudaGraphExecDestroy(H->pass_graph);
      H->pass_graph = nullptr;
    }
    if (!H->pass_graph) {
      cudaGraph_t g = nullptr;
      if ((e = cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal))) {
        H->lists_override = nullptr;
        return cuda_fail(hd, e, "capture");
      }
      cudaError_t e2 = pass();
      e = cudaStreamEndCapture(st, &g);
      if (e2 || e || (e = cudaGraphInstantiate(&H->pass_graph, g, 0))) {
        if (g) cudaGraphDestroy(g);
        H->lists_override = nullptr;
        return cuda_fail(hd, e2 ? e2 : e, "pass graph");
      }
      cudaGraphDestroy(g);
      H->pass_graph_rows = n_rows;
    }
    std::vector<cudaEvent_t> ev(iters + 1);
    for (auto& x : ev) cudaEventCreate(&x);
    cudaEventRecord(ev[0], st);
    for (int k = 0; k < iters && !rc; ++k) {
      if ((e = cudaGraphLaunch(H->pass_graph, st))) rc = cuda_fail(hd, e, "pass replay");
      cudaEventRecord(ev[k + 1], st);
    }
    if (!rc && (e = cudaStreamSynchronize(st))) rc = cuda_fail(hd, e, "pass sync");
    if (!rc && h_ms)
      for (int k = 0; k < iters; ++k) cudaEventElapsedTime(&h_ms[k], ev[k], ev[k + 1]);
    for (auto& x : ev) cudaEventDestroy(x);
  }
  H->lists_override = nullptr;
  if (rc) return rc;
  if ((e = cudaMemcpyAsync(d_hidden, H->h, (size_t)n_rows * d * 4, cudaMemcpyDeviceToDevice, st)) ||
      (e = cudaStreamSynchronize(st)))
    return cuda_fail(hd, e, "block pass result");
  Ctl c;
  return read_ctl(hd, &c);
}
