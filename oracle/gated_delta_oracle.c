/*
 * fp64 CPU oracle of the gated delta rule -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg load
 * this library.  It shares no code, header, table or helper with the CUDA
 * library; the two meet only through the seeded inputs.
 *
 * What it computes (token by token, strictly sequential, fp64):
 *
 *   thethings.ai "The argument, in one page", table "Everything, in one
 *   table", row "KDA":            S <- Diag(a) (I - beta k k^T) S + beta k v^T
 *   row "Gated DeltaNet":        S <- alpha (I - beta k k^T) S + beta k v^T
 *   row "Delta rule":            S <- (I - beta k k^T) S + beta k v^T
 *   row "Linear attention":      S += k v^T,  S in R^{d_k x d_v}
 *
 * The pages write keys as row vectors (k^T k is the d_k x d_k outer product);
 * here keys are column vectors, so the same operator reads k k^T.  The state
 * is d_k x d_v, row i belongs to key channel i (ai-explained "The efficiency
 * lineage", item 10: every row of the state gets its own lifetime).
 *
 * Readings of the pages taken here (each one is a choice the text leaves
 * open):
 *   - the gate is given as a log-decay g <= 0, a = exp(g), applied at the
 *     token it belongs to;
 *   - literal order (default): erase from the old state, then decay, then add
 *     the undecayed write -- exactly the operator order of the KDA row;
 *     the other order (decay, then erase against the decayed state) is kept
 *     as a variant;
 *   - the output reads the state after the token's own update: o_t = S_t^T q_t,
 *     with no normaliser and no 1/sqrt(d_k) scale;
 *   - with H_qk < H_v query/key heads, v-head h uses q/k head h / (H_v/H_qk).
 *
 * `mutation` exists only so that the test suite can show that its pins catch
 * plausible mistakes; 0 is the real operator.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_ERASE_THEN_DECAY 0
#define ORACLE_DECAY_THEN_ERASE 1

#define ORACLE_RULE_DELTA 0   /* rank-one erase, then write            */
#define ORACLE_RULE_LINEAR 1  /* no erase term: gated linear attention */

/* test-only planted mistakes */
#define MUT_NONE 0
#define MUT_DROP_ERASE 1       /* forget the erase term                     */
#define MUT_ERASE_SIGN 2       /* add instead of subtract the erase term    */
#define MUT_GATE_LATE 3        /* use the previous token's gate             */
#define MUT_READ_BEFORE 4      /* read out before the token's update        */
#define MUT_READ_TRANSPOSED 5  /* o_j = sum_i S[j][i] q_i (needs d_k == d_v) */
#define MUT_WRITE_NO_BETA 6    /* write k v^T without beta                  */
#define MUT_DECAY_WRITE 7      /* decay the fresh write as well             */
#define MUT_READ_WITH_KEY 8    /* read out with k instead of q              */
#define MUT_GATE_CHANNEL 9     /* per-channel gate indexed by d_k - 1 - c   */

typedef struct {
  const double *q, *k, *v, *g, *beta, *s0;
  double *o, *sT;
  const int64_t *offsets;
  int64_t num_seqs, H_qk, H_v, d_k, d_v;
  int gate_per_channel, order, rule, mutation;
  int64_t chain_begin, chain_end;
  int status;
} oracle_job;

static void run_chain(const oracle_job *J, int64_t chain, double *S, double *r, double *a) {
  const int64_t n = chain / J->H_v, h = chain % J->H_v;
  const int64_t group = J->H_v / J->H_qk, hk = h / group;
  const int64_t dk = J->d_k, dv = J->d_v;
  const int64_t bos = J->offsets[n], eos = J->offsets[n + 1];

  if (J->s0)
    memcpy(S, J->s0 + (n * J->H_v + h) * dk * dv, sizeof(double) * dk * dv);
  else
    memset(S, 0, sizeof(double) * dk * dv);

  for (int64_t t = bos; t < eos; ++t) {
    const double *qt = J->q + (t * J->H_qk + hk) * dk;
    const double *kt = J->k + (t * J->H_qk + hk) * dk;
    const double *vt = J->v + (t * J->H_v + h) * dv;
    const double b = J->beta[t * J->H_v + h];
    double *ot = J->o + (t * J->H_v + h) * dv;

    /* gate of this token: a_i = exp(g_t[i]) */
    int64_t tg = t;
    if (J->mutation == MUT_GATE_LATE) tg = (t > bos) ? t - 1 : -1;
    for (int64_t i = 0; i < dk; ++i) {
      if (tg < 0) { a[i] = 1.0; continue; }
      int64_t ci = (J->mutation == MUT_GATE_CHANNEL) ? (dk - 1 - i) : i;
      double gi = J->gate_per_channel ? J->g[(tg * J->H_v + h) * dk + ci] : J->g[tg * J->H_v + h];
      a[i] = exp(gi);
    }

    if (J->mutation == MUT_READ_BEFORE) {
      for (int64_t j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int64_t i = 0; i < dk; ++i) acc += qt[i] * S[i * dv + j];
        ot[j] = acc;
      }
    }

    if (J->order == ORACLE_DECAY_THEN_ERASE) {
      for (int64_t i = 0; i < dk; ++i)
        for (int64_t j = 0; j < dv; ++j) S[i * dv + j] *= a[i];
    }

    /* recall of the key against the state it is about to erase: r = S^T k */
    for (int64_t j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int64_t i = 0; i < dk; ++i) acc += kt[i] * S[i * dv + j];
      r[j] = acc;
    }

    const int erase = (J->rule == ORACLE_RULE_DELTA) && (J->mutation != MUT_DROP_ERASE);
    const double esign = (J->mutation == MUT_ERASE_SIGN) ? 1.0 : -1.0;
    const double wb = (J->mutation == MUT_WRITE_NO_BETA) ? 1.0 : b;
    for (int64_t i = 0; i < dk; ++i) {
      for (int64_t j = 0; j < dv; ++j) {
        double s = S[i * dv + j];
        if (erase) s = s + esign * b * kt[i] * r[j];
        if (J->order == ORACLE_ERASE_THEN_DECAY) {
          if (J->mutation == MUT_DECAY_WRITE)
            s = a[i] * (s + wb * kt[i] * vt[j]);
          else
            s = a[i] * s + wb * kt[i] * vt[j];
        } else {
          s = s + wb * kt[i] * vt[j];
        }
        S[i * dv + j] = s;
      }
    }

    if (J->mutation != MUT_READ_BEFORE) {
      const double *rq = (J->mutation == MUT_READ_WITH_KEY) ? kt : qt;
      for (int64_t j = 0; j < dv; ++j) {
        double acc = 0.0;
        if (J->mutation == MUT_READ_TRANSPOSED && dk == dv) {
          for (int64_t i = 0; i < dk; ++i) acc += rq[i] * S[j * dv + i];
        } else {
          for (int64_t i = 0; i < dk; ++i) acc += rq[i] * S[i * dv + j];
        }
        ot[j] = acc;
      }
    }
  }

  if (J->sT) memcpy(J->sT + (n * J->H_v + h) * dk * dv, S, sizeof(double) * dk * dv);
}

static void *worker(void *arg) {
  oracle_job *J = (oracle_job *)arg;
  double *S = (double *)malloc(sizeof(double) * J->d_k * J->d_v);
  double *r = (double *)malloc(sizeof(double) * J->d_v);
  double *a = (double *)malloc(sizeof(double) * J->d_k);
  if (!S || !r || !a) {
    J->status = 2;
  } else {
    for (int64_t c = J->chain_begin; c < J->chain_end; ++c) run_chain(J, c, S, r, a);
  }
  free(S);
  free(r);
  free(a);
  return NULL;
}

/*
 * Run the recurrence over every (sequence, v-head) chain.
 *
 *   q, k           [Ttot, H_qk, d_k]      tokens of all sequences, packed
 *   v              [Ttot, H_v, d_v]
 *   g              [Ttot, H_v, d_k] (gate_per_channel) or [Ttot, H_v]; log-decay
 *   beta           [Ttot, H_v]
 *   initial_state  [num_seqs, H_v, d_k, d_v] or NULL (zeros)
 *   o              [Ttot, H_v, d_v]   (output)
 *   final_state    [num_seqs, H_v, d_k, d_v] or NULL
 *   offsets        [num_seqs + 1] token offsets, non-decreasing, offsets[0] = 0
 *
 * Returns 0 on success, 1 on a bad argument, 2 on allocation failure.
 */
int oracle_gated_delta(const double *q, const double *k, const double *v, const double *g,
                       int gate_per_channel, const double *beta, const double *initial_state,
                       double *o, double *final_state, const int64_t *offsets, int64_t num_seqs,
                       int64_t H_qk, int64_t H_v, int64_t d_k, int64_t d_v, int order, int rule,
                       int mutation, int num_threads) {
  if (!q || !k || !v || !g || !beta || !o || !offsets) return 1;
  if (num_seqs < 0 || H_qk <= 0 || H_v <= 0 || d_k <= 0 || d_v <= 0) return 1;
  if (H_v % H_qk != 0) return 1;
  if (order != ORACLE_ERASE_THEN_DECAY && order != ORACLE_DECAY_THEN_ERASE) return 1;
  if (rule != ORACLE_RULE_DELTA && rule != ORACLE_RULE_LINEAR) return 1;
  if (offsets[0] != 0) return 1;
  for (int64_t n = 0; n < num_seqs; ++n)
    if (offsets[n + 1] < offsets[n]) return 1;

  const int64_t chains = num_seqs * H_v;
  if (chains == 0) return 0;
  if (num_threads < 1) num_threads = 1;
  if (num_threads > chains) num_threads = (int)chains;

  oracle_job *jobs = (oracle_job *)calloc((size_t)num_threads, sizeof(oracle_job));
  pthread_t *th = (pthread_t *)calloc((size_t)num_threads, sizeof(pthread_t));
  if (!jobs || !th) {
    free(jobs);
    free(th);
    return 2;
  }
  int status = 0;
  for (int w = 0; w < num_threads; ++w) {
    oracle_job *J = &jobs[w];
    J->q = q; J->k = k; J->v = v; J->g = g; J->beta = beta; J->s0 = initial_state;
    J->o = o; J->sT = final_state; J->offsets = offsets; J->num_seqs = num_seqs;
    J->H_qk = H_qk; J->H_v = H_v; J->d_k = d_k; J->d_v = d_v;
    J->gate_per_channel = gate_per_channel; J->order = order; J->rule = rule;
    J->mutation = mutation;
    J->chain_begin = chains * w / num_threads;
    J->chain_end = chains * (w + 1) / num_threads;
  }
  int started = 0;
  for (int w = 1; w < num_threads; ++w) {
    if (pthread_create(&th[w], NULL, worker, &jobs[w]) != 0) {
      jobs[w].status = -1; /* run it on this thread below */
    } else {
      ++started;
    }
  }
  worker(&jobs[0]);
  for (int w = 1; w < num_threads; ++w) {
    if (jobs[w].status == -1) {
      jobs[w].status = 0;
      worker(&jobs[w]);
    } else {
      pthread_join(th[w], NULL);
    }
  }
  (void)started;
  for (int w = 0; w < num_threads; ++w)
    if (jobs[w].status) status = jobs[w].status;
  free(jobs);
  free(th);
  return status;
}
