/*
 * ddt_oracle.c -- plain, slow, fp64 CPU oracle for the DDTree verification round.
 *
 * TEST INFRASTRUCTURE.  Only the test-suite, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py load this library.  The product
 * (libddt.so and its Python binding) never calls it and shares no code,
 * header, table or helper with it.
 *
 * What it computes follows the DDTree (Diffusion Draft Tree) page, a
 * curated summary of the authors' announcement:
 *   - section "運作流程" (workflow), step 1: the drafter gives one marginal
 *     q_i per position i = 1..L, conditioned only on the previous block;
 *   - section "核心創新" (core innovation) and step 2: under a node budget B
 *     the tree is the set of B most probable prefixes of the factorised
 *     draft, chosen best-first; section "理論基礎" (theory), Proposition 2:
 *     these prefixes are prefix-closed (a valid tree) and optimal;
 *     Proposition 1: the objective (expected acceptance length) is the sum
 *     of the selected prefix probabilities;
 *   - step 3: the tree is compiled to target inputs and scored in one pass
 *     with an ancestor-only attention mask ("核心創新", third bullet);
 *   - step 4: the tree walk follows the target's decoding rule, accepts a
 *     child whose token matches, and carries the first mismatch forward as
 *     the next round's bonus token: greedily (ddto_tree_walk), by sampling
 *     at a temperature (ddto_tree_walk_sample: inversion of softmax(z/T)
 *     in fp64 with a Philox4x64-10 uniform), or over row tokens
 *     already decided (ddto_walk_row_tokens, e.g. an LM head's argmax);
 *   - after step 4: the root's and the accepted rows' K/V join the committed
 *     context (ddto_kv_commit).
 *
 * Readings where the page is silent (each restated in the design notes):
 *   - candidates at depth i are the top-k tokens of q_i by (logit desc,
 *     token id asc); the tree is the best B prefixes of their product;
 *   - B counts draft nodes; the bonus token is an extra root (row 0);
 *   - total order K on prefixes: at equal depth, larger exact sum of raw
 *     logits first, then reverse-lexicographic token ids (own token,
 *     parent's token, ...); at different depths, larger fp64 score
 *     invT*sum(z) - sum(lse) first, then the shallower prefix;
 *   - compiled order is breadth-first: (depth, parent row, child rank);
 *   - the greedy walk breaks argmax ties by the lowest token id.
 *
 * All arithmetic is fp64.  Inputs arrive as bf16 (raw uint16 bits) or f32
 * and are widened exactly.  Compile with -ffp-contract=off so that every
 * product and sum is rounded as written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define DDTO_LMAX 64
#define DDTO_OK 0
#define DDTO_ERR_ARG 1
#define DDTO_ERR_NOMEM 2

/* ------------------------------------------------------------------ */
/* value widening                                                      */
/* ------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE binary32; widening is a shift. */
static double bf16_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double load_val(const void* base, int is_bf16, int64_t idx) {
  if (is_bf16) return bf16_to_double(((const uint16_t*)base)[idx]);
  return (double)((const float*)base)[idx];
}

/* ------------------------------------------------------------------ */
/* Step 1: softmax (log-sum-exp) and per-position top-k                */
/* ------------------------------------------------------------------ */

typedef struct {
  double z;
  int32_t id;
} zid_t;

/* (z desc, id asc): the candidate order at one position. */
static int cmp_zid(const void* pa, const void* pb) {
  const zid_t* a = (const zid_t*)pa;
  const zid_t* b = (const zid_t*)pb;
  if (a->z > b->z) return -1;
  if (a->z < b->z) return 1;
  return (a->id < b->id) ? -1 : (a->id > b->id);
}

/*
 * For each of `rows` rows of V logits z (row r starts at r*row_stride):
 *   u = invT * z,  lse = log sum_v exp(u_v)  (max-shifted),
 *   the k tokens with the largest z (ties: smaller id first), their raw z,
 *   and logp = invT * z - lse.
 * The candidate order is decided on the raw z, so a positive temperature
 * cannot reorder it.  Full sort of the row: slow and obviously correct.
 */
int ddto_topk(const void* z, int is_bf16, int rows, int V, int64_t row_stride, int k,
              double invT, int32_t* ids, double* zk, double* logp, double* lse) {
  if (!z || rows < 0 || V < 1 || k < 1 || k > V || row_stride < V || !(invT > 0.0))
    return DDTO_ERR_ARG;
  zid_t* buf = (zid_t*)malloc(sizeof(zid_t) * (size_t)V);
  if (!buf) return DDTO_ERR_NOMEM;
  for (int r = 0; r < rows; ++r) {
    const int64_t base = (int64_t)r * row_stride;
    double m = -INFINITY;
    for (int v = 0; v < V; ++v) {
      buf[v].z = load_val(z, is_bf16, base + v);
      buf[v].id = v;
      double u = invT * buf[v].z;
      if (u > m) m = u;
    }
    double s = 0.0;
    for (int v = 0; v < V; ++v) s += exp(invT * buf[v].z - m);
    const double row_lse = m + log(s);
    qsort(buf, (size_t)V, sizeof(zid_t), cmp_zid);
    for (int j = 0; j < k; ++j) {
      ids[(int64_t)r * k + j] = buf[j].id;
      zk[(int64_t)r * k + j] = buf[j].z;
      logp[(int64_t)r * k + j] = invT * buf[j].z - row_lse;
    }
    lse[r] = row_lse;
  }
  free(buf);
  return DDTO_OK;
}

/* ------------------------------------------------------------------ */
/* Step 2: the B best prefixes of the factorised draft                 */
/* ------------------------------------------------------------------ */

typedef struct {
  int depth;                 /* number of drafted positions, 1..L */
  int16_t r[DDTO_LMAX];      /* rank at each position (index into top-k list) */
  double sz;                 /* exact sum of raw logits along the prefix */
  double score;              /* invT * sz - S[depth]: log-probability of the prefix */
} pfx_t;

typedef struct {
  int L, k, kstride;
  double invT;
  const int32_t* ids;        /* [L][kstride] */
  const double* zk;          /* [L][kstride] */
  double S[DDTO_LMAX + 1];   /* S[t] = lse_1 + ... + lse_t, summed left to right */
} tctx_t;

static int32_t tok_at(const tctx_t* c, int pos, int rank) {
  return c->ids[(int64_t)pos * c->kstride + rank];
}

/* score of a prefix of depth t with logit sum sz: invT*sz - S[t]. */
static double prefix_score(const tctx_t* c, int t, double sz) {
  double a = c->invT * sz;
  return a - c->S[t];
}

/* The total order K.  Returns <0 if a precedes b (is the better prefix). */
static int k_cmp(const tctx_t* c, const pfx_t* a, const pfx_t* b) {
  if (a->depth == b->depth) {
    /* equal depth: the shared sum of lse cancels, compare exact logit sums */
    if (a->sz > b->sz) return -1;
    if (a->sz < b->sz) return 1;
    for (int i = a->depth - 1; i >= 0; --i) {
      int32_t ta = tok_at(c, i, a->r[i]);
      int32_t tb = tok_at(c, i, b->r[i]);
      if (ta != tb) return (ta < tb) ? -1 : 1;
    }
    return 0;
  }
  if (a->score > b->score) return -1;
  if (a->score < b->score) return 1;
  return (a->depth < b->depth) ? -1 : 1;
}

typedef struct {
  const tctx_t* c;
  pfx_t* best;   /* current best set, at most B entries, unordered */
  int n, B;
  int worst;     /* index of the K-last entry of best[] when n == B */
} bestset_t;

static void bestset_find_worst(bestset_t* s) {
  int w = 0;
  for (int i = 1; i < s->n; ++i)
    if (k_cmp(s->c, &s->best[i], &s->best[w]) > 0) w = i;
  s->worst = w;
}

/* Would prefix p enter the current best set? */
static int bestset_admits(const bestset_t* s, const pfx_t* p) {
  if (s->n < s->B) return 1;
  return k_cmp(s->c, p, &s->best[s->worst]) < 0;
}

static void bestset_insert(bestset_t* s, const pfx_t* p) {
  if (s->n < s->B) {
    s->best[s->n++] = *p;
    if (s->n == s->B) bestset_find_worst(s);
  } else {
    s->best[s->worst] = *p;
    bestset_find_worst(s);
  }
}

/*
 * Depth-first enumeration of every prefix, with monotone pruning.
 * A child never precedes its parent under K (its log-probability is no
 * larger and it is deeper), and a later sibling never precedes an earlier
 * one (the candidate list is in K order).  So once a prefix fails to enter
 * the current best-B set, neither its subtree nor its later siblings can.
 */
static void enumerate(bestset_t* s, const pfx_t* parent) {
  const tctx_t* c = s->c;
  if (parent->depth >= c->L) return;
  const int pos = parent->depth;  /* 0-based position of the children */
  for (int r = 0; r < c->k; ++r) {
    pfx_t ch = *parent;
    ch.depth = parent->depth + 1;
    ch.r[pos] = (int16_t)r;
    ch.sz = parent->sz + c->zk[(int64_t)pos * c->kstride + r];
    ch.score = prefix_score(c, ch.depth, ch.sz);
    if (!bestset_admits(s, &ch)) break;
    bestset_insert(s, &ch);
    enumerate(s, &ch);
  }
}

/* is prefix a the parent of prefix b? */
static int is_parent_of(const pfx_t* a, const pfx_t* b) {
  if (b->depth != a->depth + 1) return 0;
  for (int i = 0; i < a->depth; ++i)
    if (a->r[i] != b->r[i]) return 0;
  return 1;
}

/*
 * Build and compile the tree of one sequence.
 *   ids, zk: [L][kstride] top-k ids and raw logits (k <= kstride used);
 *   lse: [L] per-position log-sum-exp;  B: draft-node budget;
 *   Nmax: rows in the output tensors (>= B+1);  W: mask words per row.
 * Outputs (rows >= n_nodes are padding: -1 / 0):
 *   tok, parent, depth, pos [Nmax], mask [Nmax][W] (bit i of row j set iff
 *   node i is node j or one of its ancestors), n_nodes, surrogate
 *   (sum over draft nodes of exp(score)), delta_min (smallest |score gap|
 *   between a selected node and an unselected child of the tree at a
 *   different depth; +inf if there is none).
 */
int ddto_build_tree(int L, int k, int kstride, int B, double invT, const int32_t* ids,
                    const double* zk, const double* lse, int32_t root_token, int32_t ctx_len,
                    int Nmax, int W, int32_t* tok, int32_t* parent, int32_t* depth, int32_t* pos,
                    uint32_t* mask, int32_t* n_nodes, double* surrogate, double* delta_min) {
  if (L < 1 || L > DDTO_LMAX || k < 1 || k > kstride || B < 0 || Nmax < B + 1 ||
      W * 32 < Nmax || !(invT > 0.0))
    return DDTO_ERR_ARG;
  tctx_t c;
  c.L = L;
  c.k = k;
  c.kstride = kstride;
  c.invT = invT;
  c.ids = ids;
  c.zk = zk;
  c.S[0] = 0.0;
  for (int t = 1; t <= L; ++t) c.S[t] = c.S[t - 1] + lse[t - 1];

  bestset_t s;
  s.c = &c;
  s.B = B;
  s.n = 0;
  s.worst = 0;
  s.best = (pfx_t*)malloc(sizeof(pfx_t) * (size_t)(B > 0 ? B : 1));
  if (!s.best) return DDTO_ERR_NOMEM;
  pfx_t root;
  memset(&root, 0, sizeof root);
  if (B > 0) enumerate(&s, &root);
  const int nsel = s.n;

  /* Compile: breadth-first order by (depth, parent row, child rank). */
  pfx_t* rows = (pfx_t*)malloc(sizeof(pfx_t) * (size_t)(nsel + 1));
  int* used = (int*)calloc((size_t)(nsel > 0 ? nsel : 1), sizeof(int));
  if (!rows || !used) {
    free(s.best);
    free(rows);
    free(used);
    return DDTO_ERR_NOMEM;
  }
  rows[0] = root;
  int nrow = 1;
  for (int i = 0; i < Nmax; ++i) {
    tok[i] = -1;
    parent[i] = -1;
    depth[i] = -1;
    pos[i] = -1;
  }
  memset(mask, 0, sizeof(uint32_t) * (size_t)Nmax * (size_t)W);
  tok[0] = root_token;
  depth[0] = 0;
  pos[0] = ctx_len;
  for (int head = 0; head < nrow; ++head) {
    /* children of row `head`, in increasing rank */
    for (int r = 0; r < k; ++r) {
      for (int i = 0; i < nsel; ++i) {
        if (used[i]) continue;
        const pfx_t* p = &s.best[i];
        if (is_parent_of(&rows[head], p) && p->r[p->depth - 1] == r) {
          used[i] = 1;
          rows[nrow] = *p;
          tok[nrow] = tok_at(&c, p->depth - 1, r);
          parent[nrow] = head;
          depth[nrow] = p->depth;
          pos[nrow] = ctx_len + p->depth;
          ++nrow;
        }
      }
    }
  }
  /* every selected prefix must have been reached from the root */
  const int closed = (nrow == nsel + 1);
  /* ancestor-or-self sets by walking parent pointers */
  for (int j = 0; j < nrow; ++j)
    for (int a = j; a >= 0; a = parent[a]) mask[(int64_t)j * W + a / 32] |= 1u << (a % 32);

  double surr = 0.0;
  for (int j = 1; j < nrow; ++j) surr += exp(rows[j].score);

  /* margin: selected vs unselected children of the tree, at other depths */
  double dmin = INFINITY;
  for (int x = 0; x < nrow; ++x) {
    if (rows[x].depth >= L) continue;
    for (int r = 0; r < k; ++r) {
      pfx_t ch = rows[x];
      ch.depth = rows[x].depth + 1;
      ch.r[rows[x].depth] = (int16_t)r;
      ch.sz = rows[x].sz + zk[(int64_t)rows[x].depth * kstride + r];
      ch.score = prefix_score(&c, ch.depth, ch.sz);
      int selected = 0;
      for (int j = 1; j < nrow && !selected; ++j)
        if (rows[j].depth == ch.depth && is_parent_of(&rows[x], &rows[j]) &&
            rows[j].r[ch.depth - 1] == r)
          selected = 1;
      if (selected) continue;
      for (int j = 1; j < nrow; ++j) {
        if (rows[j].depth == ch.depth) continue;
        double g = fabs(rows[j].score - ch.score);
        if (g < dmin) dmin = g;
      }
    }
  }

  *n_nodes = nrow;
  *surrogate = surr;
  *delta_min = dmin;
  free(s.best);
  free(rows);
  free(used);
  return closed ? DDTO_OK : DDTO_ERR_ARG;
}

/* ------------------------------------------------------------------ */
/* Step 3: masked attention of every tree row                          */
/* ------------------------------------------------------------------ */

/*
 * For each requested item (b, j, h): the attention output of tree row j,
 * query head h of sequence b, over the sequence's committed context
 * (positions 0..ctx_len[b]-1) and the tree rows i whose mask bit (j, i) is
 * set (ancestors-or-self).  Scores are scale * <q, k>; softmax in fp64.
 *
 * Layouts (bf16 raw bits): q [batch][Nmax][Hq][d];
 *   dense cache (page_table == NULL): k/v [batch][Tmax][Hkv][d];
 *   paged cache: k/v [pages][page_size][Hkv][d] with the context position t
 *   of sequence b at page page_table[b*max_pages + t/page_size], slot
 *   t % page_size;
 *   tree k/v [batch][Nmax][Hkv][d]; mask [batch][Nmax][W].
 * Query head h reads kv head h / (Hq/Hkv).
 * Outputs: out [n_items][d], lse_out [n_items] (natural log of the softmax
 * normaliser, in units of the scaled score).
 */
int ddto_tree_attn(int n_items, const int32_t* items, const uint16_t* q, int Nmax, int Hq,
                   int Hkv, int d, const uint16_t* k_cache, const uint16_t* v_cache,
                   int64_t Tmax, const int32_t* page_table, int page_size, int max_pages,
                   const int32_t* ctx_len, const uint16_t* k_tree, const uint16_t* v_tree,
                   const uint32_t* mask, int W, const int32_t* n_nodes, double scale,
                   double* out, double* lse_out) {
  if (n_items < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || d < 1) return DDTO_ERR_ARG;
  const int g = Hq / Hkv;
  int64_t max_ctx = 0;
  for (int it = 0; it < n_items; ++it) {
    int b = items[3 * it];
    if (ctx_len[b] > max_ctx) max_ctx = ctx_len[b];
  }
  double* sc = (double*)malloc(sizeof(double) * (size_t)(max_ctx + Nmax + 1));
  double* qv = (double*)malloc(sizeof(double) * (size_t)d);
  if (!sc || !qv) {
    free(sc);
    free(qv);
    return DDTO_ERR_NOMEM;
  }
  for (int it = 0; it < n_items; ++it) {
    const int b = items[3 * it], j = items[3 * it + 1], h = items[3 * it + 2];
    const int kvh = h / g;
    const int T = ctx_len[b];
    const int n = n_nodes[b];
    double* o = out + (int64_t)it * d;
    for (int e = 0; e < d; ++e) {
      qv[e] = bf16_to_double(q[(((int64_t)b * Nmax + j) * Hq + h) * d + e]);
      o[e] = 0.0;
    }
    if (j >= n) {
      lse_out[it] = -INFINITY;
      continue;
    }
    /* scores */
    double m = -INFINITY;
    int nsc = 0;
    for (int t = 0; t < T; ++t) {
      int64_t row;
      if (page_table)
        row = ((int64_t)page_table[(int64_t)b * max_pages + t / page_size] * page_size +
               t % page_size);
      else
        row = (int64_t)b * Tmax + t;
      const uint16_t* kp = k_cache + (row * Hkv + kvh) * d;
      double dot = 0.0;
      for (int e = 0; e < d; ++e) dot += qv[e] * bf16_to_double(kp[e]);
      sc[nsc] = scale * dot;
      if (sc[nsc] > m) m = sc[nsc];
      ++nsc;
    }
    for (int i = 0; i < n; ++i) {
      const int vis = (mask[((int64_t)b * Nmax + j) * W + i / 32] >> (i % 32)) & 1u;
      if (!vis) continue;
      const uint16_t* kp = k_tree + (((int64_t)b * Nmax + i) * Hkv + kvh) * d;
      double dot = 0.0;
      for (int e = 0; e < d; ++e) dot += qv[e] * bf16_to_double(kp[e]);
      sc[nsc] = scale * dot;
      if (sc[nsc] > m) m = sc[nsc];
      ++nsc;
    }
    /* softmax-weighted sum of values, same visiting order */
    double l = 0.0;
    int c = 0;
    for (int t = 0; t < T; ++t, ++c) {
      int64_t row;
      if (page_table)
        row = ((int64_t)page_table[(int64_t)b * max_pages + t / page_size] * page_size +
               t % page_size);
      else
        row = (int64_t)b * Tmax + t;
      const uint16_t* vp = v_cache + (row * Hkv + kvh) * d;
      const double p = exp(sc[c] - m);
      l += p;
      for (int e = 0; e < d; ++e) o[e] += p * bf16_to_double(vp[e]);
    }
    for (int i = 0; i < n; ++i) {
      const int vis = (mask[((int64_t)b * Nmax + j) * W + i / 32] >> (i % 32)) & 1u;
      if (!vis) continue;
      const uint16_t* vp = v_tree + (((int64_t)b * Nmax + i) * Hkv + kvh) * d;
      const double p = exp(sc[c] - m);
      ++c;
      l += p;
      for (int e = 0; e < d; ++e) o[e] += p * bf16_to_double(vp[e]);
    }
    for (int e = 0; e < d; ++e) o[e] /= l;
    lse_out[it] = m + log(l);
  }
  free(sc);
  free(qv);
  return DDTO_OK;
}

/* ------------------------------------------------------------------ */
/* Step 4: greedy tree walk                                            */
/* ------------------------------------------------------------------ */

/*
 * Greedy walk of one sequence's tree over its target logits
 * (row j at logits + j*row_stride, V entries, bf16 or f32).
 * From the root: t = argmax of the current row (lowest id on ties); if the
 * current node has a child carrying t, accept it and descend; otherwise t
 * is the bonus token and the walk stops.
 * acc_nodes / acc_tok receive L entries (unused ones -1).
 */
int ddto_tree_walk(const void* logits, int is_bf16, int64_t row_stride, int V,
                   const int32_t* tok, const int32_t* parent, const int32_t* depth, int n_nodes,
                   int L, int32_t* acc_len, int32_t* acc_nodes, int32_t* acc_tok,
                   int32_t* bonus) {
  if (!logits || V < 1 || n_nodes < 1 || L < 0) return DDTO_ERR_ARG;
  for (int i = 0; i < L; ++i) {
    acc_nodes[i] = -1;
    acc_tok[i] = -1;
  }
  int x = 0, a = 0;
  for (;;) {
    const int64_t base = (int64_t)x * row_stride;
    int best = 0;
    double bv = load_val(logits, is_bf16, base);
    for (int v = 1; v < V; ++v) {
      double val = load_val(logits, is_bf16, base + v);
      if (val > bv) {
        bv = val;
        best = v;
      }
    }
    int next = -1;
    if (depth[x] < L)
      for (int c = 0; c < n_nodes; ++c)
        if (parent[c] == x && tok[c] == best) {
          next = c;
          break;
        }
    if (next < 0 || a >= L) {
      *bonus = best;
      break;
    }
    acc_nodes[a] = next;
    acc_tok[a] = best;
    ++a;
    x = next;
  }
  *acc_len = a;
  return DDTO_OK;
}

/* ------------------------------------------------------------------ */
/* Sampled walk (target temperature > 0)                               */
/* ------------------------------------------------------------------ */
/*
 * Step 4 says the walk follows the target's decoding rule; the announcement
 * reports results over several temperatures, so besides greedy decoding the
 * rule may be sampling from softmax(z / T).  The walk stays lossless when
 * each visited row draws its token from that distribution with a fresh
 * uniform: every emitted token is then a draw from the target's conditional
 * given the accepted prefix, exactly as if the target had decoded alone.
 *
 * Reading adopted (the page gives no sampler): inverse-CDF sampling over
 * token ids in increasing order, one uniform u per (sequence, tree row),
 * u taken from the counter-based generator Philox4x64-10 so that any
 * implementation can reproduce the draw.
 */

/* 64 x 64 -> 128-bit product, split into high and low words. */
static void mulhilo64(uint64_t a, uint64_t b, uint64_t* hi, uint64_t* lo) {
  const unsigned __int128 p = (unsigned __int128)a * (unsigned __int128)b;
  *hi = (uint64_t)(p >> 64);
  *lo = (uint64_t)p;
}

/*
 * Philox4x64-10 (Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers:
 * As Easy as 1, 2, 3", SC'11, section 4).  One round: words 0 and 2 of the
 * counter are multiplied by the two round multipliers; the new word 0 is
 * the high half of the second product xor word 1 xor key word 0, the new
 * word 2 is the high half of the first product xor word 3 xor key word 1,
 * and the low halves become words 1 and 3.  Between rounds the key words
 * advance by the two Weyl increments (golden ratio and sqrt(3) - 1, as
 * 64-bit fractions).  Ten rounds.
 */
void ddto_philox4x64_10(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4]) {
  const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
  const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
  uint64_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
  uint64_t k0 = key[0], k1 = key[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += W0;
      k1 += W1;
    }
    uint64_t hi0, lo0, hi1, lo1;
    mulhilo64(M0, x0, &hi0, &lo0);
    mulhilo64(M1, x2, &hi1, &lo1);
    const uint64_t n0 = hi1 ^ x1 ^ k0, n2 = hi0 ^ x3 ^ k1;
    x0 = n0;
    x1 = lo1;
    x2 = n2;
    x3 = lo0;
  }
  out[0] = x0;
  out[1] = x1;
  out[2] = x2;
  out[3] = x3;
}

/* A 64-bit word to a uniform in (0, 1): its top 52 bits, centred in their
   interval of width 2^-52.  Every value is exact in binary64 and lies in
   [2^-53, 1 - 2^-53], so it is never 0 and never 1. */
double ddto_word_to_uniform(uint64_t w) {
  return ((double)(w >> 12) + 0.5) * 0x1.0p-52;
}

/* The uniform of tree row j of sequence b in the round numbered `step`:
   word 0 of Philox4x64-10 at counter (j, b, 0, 0) under key (seed, step). */
double ddto_row_uniform(uint64_t seed, uint64_t step, int b, int j) {
  const uint64_t ctr[4] = {(uint64_t)(uint32_t)j, (uint64_t)(uint32_t)b, 0, 0};
  const uint64_t key[2] = {seed, step};
  uint64_t out[4];
  ddto_philox4x64_10(ctr, key, out);
  return ddto_word_to_uniform(out[0]);
}

/*
 * The draw's weights: the target's distribution softmax(invT * z) before
 * normalisation, in fp64.  With m = max_v invT * z_v over the finite
 * logits, w_v = exp(invT * z_v - m); a -inf logit weighs 0.  Returns
 * S = sum_v w_v summed in index order, or 0 when no logit is finite.
 */
static double sampler_weights(const void* logits, int is_bf16, int64_t base, int V, double invT,
                              double* w) {
  double m = -INFINITY;
  for (int v = 0; v < V; ++v) {
    const double y = invT * load_val(logits, is_bf16, base + v);
    if (y > m) m = y;
  }
  if (m == -INFINITY) {
    for (int v = 0; v < V; ++v) w[v] = 0.0;
    return 0.0;
  }
  double S = 0.0;
  for (int v = 0; v < V; ++v) {
    w[v] = exp(invT * load_val(logits, is_bf16, base + v) - m);
    S += w[v];
  }
  return S;
}

/* The weights of a row, for the tests. */
int ddto_sampler_row_weights(const void* logits, int is_bf16, int V, double invT, double* w) {
  if (!logits || V < 1 || !(invT > 0.0)) return DDTO_ERR_ARG;
  sampler_weights(logits, is_bf16, 0, V, invT, w);
  return DDTO_OK;
}

/*
 * One draw from the weights above by inversion: with S = sum w and
 * C_v = w_0 + ... + w_v (ids in increasing order), the token is the
 * smallest v with C_v > u*S.  *margin receives the distance of u*S from the
 * nearer end of the chosen interval [C_{v-1}, C_v), divided by S: a draw
 * with a margin below a computation's relative rounding error may come out
 * differently there.  A row with no finite logit yields token 0 (margin
 * +inf).
 */
int ddto_sample_row(const void* logits, int is_bf16, int64_t base, int V, double invT, double u,
                    double* margin) {
  double* w = (double*)malloc(sizeof(double) * (size_t)V);
  if (!w) return -1;
  const double S = sampler_weights(logits, is_bf16, base, V, invT, w);
  if (!(S > 0.0)) {
    free(w);
    *margin = INFINITY;
    return 0;
  }
  const double theta = u * S;
  double C = 0.0;
  int last_pos = 0;
  for (int v = 0; v < V; ++v) {
    const double prev = C;
    C += w[v];
    if (w[v] > 0.0) last_pos = v;
    if (C > theta) {
      const double d0 = theta - prev, d1 = C - theta;
      *margin = (d0 < d1 ? d0 : d1) / S;
      free(w);
      return v;
    }
  }
  free(w);
  *margin = 0.0; /* u*S rounded onto the total: the last token of positive weight */
  return last_pos;
}

/*
 * Sampled walk of sequence b: as ddto_tree_walk, but the token taken at
 * row x is ddto_sample_row(row x, invT, ddto_row_uniform(seed, step, b, x)).
 * *min_margin receives the smallest draw margin along the walk.
 */
int ddto_tree_walk_sample(const void* logits, int is_bf16, int64_t row_stride, int V,
                          const int32_t* tok, const int32_t* parent, const int32_t* depth,
                          int n_nodes, int L, double invT, uint64_t seed, uint64_t step, int b,
                          int32_t* acc_len, int32_t* acc_nodes, int32_t* acc_tok, int32_t* bonus,
                          double* min_margin) {
  if (!logits || V < 1 || n_nodes < 1 || L < 0 || !(invT > 0.0)) return DDTO_ERR_ARG;
  for (int i = 0; i < L; ++i) {
    acc_nodes[i] = -1;
    acc_tok[i] = -1;
  }
  double mm = INFINITY;
  int x = 0, a = 0;
  for (;;) {
    double mg;
    const double u = ddto_row_uniform(seed, step, b, x);
    const int t = ddto_sample_row(logits, is_bf16, (int64_t)x * row_stride, V, invT, u, &mg);
    if (mg < mm) mm = mg;
    int next = -1;
    if (depth[x] < L)
      for (int c = 0; c < n_nodes; ++c)
        if (parent[c] == x && tok[c] == t) {
          next = c;
          break;
        }
    if (next < 0 || a >= L) {
      *bonus = t;
      break;
    }
    acc_nodes[a] = next;
    acc_tok[a] = t;
    ++a;
    x = next;
  }
  *acc_len = a;
  *min_margin = mm;
  return DDTO_OK;
}

/* ------------------------------------------------------------------ */
/* KV commit of the accepted path                                      */
/* ------------------------------------------------------------------ */
/*
 * After the walk (step 4), the round has forwarded the root (the previous
 * round's bonus token, which the target had produced but not yet run; page
 * workflow, opening paragraph) and the accepted rows; the new bonus token
 * has not been forwarded.  So the committed context of sequence b grows by
 * acc_len + 1 positions: position ctx_len + i receives the K/V of the i-th
 * row of the path root, acc_nodes[0], ..., acc_nodes[acc_len - 1] (the row
 * at depth i, whose position id was ctx_len + i), and ctx_len advances by
 * acc_len + 1.
 *
 * Layouts (bf16 as raw uint16): tree K/V [n_max][hkv][d] of this sequence;
 * the cache either dense [t_max][hkv][d] of this sequence (page_table NULL)
 * or a page pool [pages][page_size][hkv][d] with this sequence's page list.
 * A position outside the cache (or a page id outside the pool) is not
 * written; the function then returns DDTO_ERR_ARG after writing the rest.
 */
int ddto_kv_commit(const uint16_t* k_tree, const uint16_t* v_tree, int n_max, int hkv, int d,
                   int acc_len, const int32_t* acc_nodes, int32_t* ctx_len, uint16_t* k_cache,
                   uint16_t* v_cache, int64_t t_max, const int32_t* pages, int page_size,
                   int max_pages, int num_pages) {
  if (!k_tree || !v_tree || !ctx_len || !k_cache || !v_cache || acc_len < 0 || hkv < 1 || d < 1)
    return DDTO_ERR_ARG;
  const int64_t row = (int64_t)hkv * d;
  const int c = *ctx_len;
  int bad = 0;
  for (int i = 0; i <= acc_len; ++i) {
    const int r = i == 0 ? 0 : acc_nodes[i - 1];
    if (r < 0 || r >= n_max) {
      bad = 1;
      continue;
    }
    const int64_t pos = (int64_t)c + i;
    int64_t dst;
    if (!pages) {
      if (pos >= t_max) {
        bad = 1;
        continue;
      }
      dst = pos * row;
    } else {
      const int64_t pi = pos / page_size;
      const int pg = pi < max_pages ? pages[pi] : -1;
      if (pg < 0 || (num_pages > 0 && pg >= num_pages)) {
        bad = 1;
        continue;
      }
      dst = ((int64_t)pg * page_size + pos % page_size) * row;
    }
    for (int64_t e = 0; e < row; ++e) {
      k_cache[dst + e] = k_tree[(int64_t)r * row + e];
      v_cache[dst + e] = v_tree[(int64_t)r * row + e];
    }
  }
  *ctx_len = c + acc_len + 1;
  return bad ? DDTO_ERR_ARG : DDTO_OK;
}

/* ------------------------------------------------------------------ */
/* Walk over given row tokens (the target's argmax of each tree row)   */
/* ------------------------------------------------------------------ */
/*
 * Step 4 when the target's decision at each row is already known (for
 * instance from an LM head whose logits are never stored): row_tok[j] is
 * the token the target emits after row j.  From the root: if the current
 * row has a child carrying that token (and depth < L), accept it and
 * continue; otherwise that token is the bonus.  Same outputs as
 * ddto_tree_walk.
 */
int ddto_walk_row_tokens(const int32_t* row_tok, const int32_t* tok, const int32_t* parent,
                         const int32_t* depth, int n_nodes, int L, int32_t* acc_len,
                         int32_t* acc_nodes, int32_t* acc_tok, int32_t* bonus) {
  if (!row_tok || n_nodes < 1 || L < 0) return DDTO_ERR_ARG;
  for (int i = 0; i < L; ++i) {
    acc_nodes[i] = -1;
    acc_tok[i] = -1;
  }
  int x = 0, a = 0;
  for (;;) {
    const int t = row_tok[x];
    int next = -1;
    if (depth[x] < L)
      for (int c = 0; c < n_nodes; ++c)
        if (parent[c] == x && tok[c] == t) {
          next = c;
          break;
        }
    if (next < 0 || a >= L) {
      *bonus = t;
      break;
    }
    acc_nodes[a] = next;
    acc_tok[a] = t;
    ++a;
    x = next;
  }
  *acc_len = a;
  return DDTO_OK;
}

/* ------------------------------------------------------------------ */
/* Node budgets across a batch (after step 2)                          */
/* ------------------------------------------------------------------ */
/*
 * The page's trade-off (section 實驗結果與權衡): a larger node budget raises
 * the expected acceptance but the verifier's cost grows with it.  By
 * Proposition 1 (section 理論基礎) a tree's expected acceptance length is the
 * sum of its nodes' prefix probabilities, and the best tree of any smaller
 * budget is the K-first part of the best tree of a larger one.  So, given
 * for every sequence the tree built with its largest budget, the nodes of
 * the whole batch ranked by prefix probability (by its logarithm, the score;
 * ties: smaller sequence index, then smaller row) give the allocation that maximises the summed
 * expected acceptance for any total number of nodes n: the first n nodes.
 * With a round cost of c0 + c1 * n for n draft nodes, the round emits
 * (batch + accepted) tokens, so the plan takes the n that maximises
 * (batch + sum of the first n probabilities) / (c0 + c1 * n) (the smallest
 * such n), up to `total_budget` nodes (< 0: no cap).  With c1 <= 0 it takes
 * all the nodes up to the cap.  Outputs: budget[b], the number of sequence
 * b's nodes among those taken, and expected_tokens[b] = 1 + the sum of their
 * probabilities (the tokens sequence b is expected to emit).
 *
 * Node probabilities: a row j of sequence b at depth d with tokens
 * t_1..t_d on its path has score invT * (z_1 + ... + z_d) - (lse_1 + ... +
 * lse_d), each sum in depth order (z_i the candidate logit of t_i at
 * position i from the top-k lists ids / zk [L][kstride], lse [L]); the
 * probability is exp(score).
 */
typedef struct {
  double score, p;
  int b, j;
} pnode_t;

/* by score (the probability's logarithm, so that no two distinct scores
   tie through the rounding of exp), then sequence, then row */
static int cmp_pnode(const void* pa, const void* pb) {
  const pnode_t* a = (const pnode_t*)pa;
  const pnode_t* b = (const pnode_t*)pb;
  if (a->score > b->score) return -1;
  if (a->score < b->score) return 1;
  if (a->b != b->b) return a->b < b->b ? -1 : 1;
  return a->j < b->j ? -1 : (a->j > b->j);
}

int ddto_plan_budget(int batch, int L, int kstride, int n_max, double invT, const int32_t* ids,
                     const double* zk, const double* lse, const int32_t* tok,
                     const int32_t* parent, const int32_t* depth, const int32_t* n_nodes,
                     int total_budget, double c0, double c1, int32_t* budget,
                     double* expected_tokens, int32_t* n_taken) {
  if (batch < 0 || L < 1 || L > DDTO_LMAX || kstride < 1 || n_max < 1 || !(invT > 0.0))
    return DDTO_ERR_ARG;
  if (c1 > 0.0 && !(c0 > 0.0)) return DDTO_ERR_ARG;
  int total = 0;
  for (int b = 0; b < batch; ++b)
    if (n_nodes[b] > 1) total += n_nodes[b] - 1;
  pnode_t* nodes = (pnode_t*)malloc(sizeof(pnode_t) * (size_t)(total > 0 ? total : 1));
  if (!nodes) return DDTO_ERR_NOMEM;
  int m = 0;
  for (int b = 0; b < batch; ++b) {
    const int32_t* bt = tok + (int64_t)b * n_max;
    const int32_t* bp = parent + (int64_t)b * n_max;
    const int32_t* bd = depth + (int64_t)b * n_max;
    for (int j = 1; j < n_nodes[b]; ++j) {
      /* the path's tokens, root excluded, from depth 1 down to depth d */
      int path[DDTO_LMAX];
      const int d = bd[j];
      if (d < 1 || d > L) {
        free(nodes);
        return DDTO_ERR_ARG;
      }
      for (int x = j, t = d; t >= 1; x = bp[x], --t) path[t - 1] = bt[x];
      double sz = 0.0, S = 0.0;
      for (int t = 0; t < d; ++t) {
        const int64_t row = ((int64_t)b * L + t) * kstride;
        int r = 0;
        while (r < kstride && ids[row + r] != path[t]) ++r;
        if (r == kstride) {
          free(nodes);
          return DDTO_ERR_ARG;
        }
        sz = sz + zk[row + r];
        S = S + lse[(int64_t)b * L + t];
      }
      const double a = invT * sz;
      nodes[m].score = a - S;
      nodes[m].p = exp(nodes[m].score);
      nodes[m].b = b;
      nodes[m].j = j;
      ++m;
    }
  }
  qsort(nodes, (size_t)m, sizeof(pnode_t), cmp_pnode);
  int cap = m;
  if (total_budget >= 0 && total_budget < cap) cap = total_budget;
  int best_n = cap;
  if (c1 > 0.0) {
    double P = 0.0, best = (double)batch / c0;
    best_n = 0;
    for (int n = 1; n <= cap; ++n) {
      P += nodes[n - 1].p;
      const double f = ((double)batch + P) / (c0 + c1 * (double)n);
      if (f > best) {
        best = f;
        best_n = n;
      }
    }
  }
  for (int b = 0; b < batch; ++b) {
    budget[b] = 0;
    expected_tokens[b] = 1.0;
  }
  for (int i = 0; i < best_n; ++i) {
    budget[nodes[i].b] += 1;
    expected_tokens[nodes[i].b] += nodes[i].p;
  }
  *n_taken = best_n;
  free(nodes);
  return DDTO_OK;
}
