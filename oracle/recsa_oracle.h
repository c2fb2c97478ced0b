/*
 * fp64 CPU oracle for RecSA tree sparse attention — TEST INFRASTRUCTURE.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg use
 * this library. It shares no code with the CUDA path.
 *
 * Method source: "Recursive Sparse Attention: Million-Token Length
 * Extrapolation at Logarithmic Cost" (arXiv 2611.07232), abstract; and the
 * kongchang.com article on RecSA, sections "Core Idea" and "Position
 * Encoding". Readings of what the pages leave open are listed in the .c file.
 *
 * Token arrays (level 0) are row-major [rows][d], either float32 or bf16 bit
 * patterns (tok_dtype 0 / 1). Node arrays are fp64 [n_j][d], one per level,
 * holding the values as stored (rounded to the storage type).
 */
#ifndef RECSA_ORACLE_H
#define RECSA_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

#define ORC_MAXLEV 40

enum { ORC_TOK_F32 = 0, ORC_TOK_BF16 = 1 };
enum { ORC_STORE_F32 = 0, ORC_STORE_BF16 = 1, ORC_STORE_F64 = 2 };

/* Level sizes of the tree over T tokens: n[0] = T, n[j] = ceil(n[j-1]/b),
 * stopping at the first j >= 1 with n[j] <= b. Returns that j (J), or 0 for
 * T == 0. n must hold ORC_MAXLEV + 1 entries; entries above J are set to 1
 * (or 0 when T == 0). */
int orc_levels(long long T, int b, long long* n);

/* Round x to the storage type (fp32, bf16 or fp64), nearest-even. */
double orc_round(double x, int storage);

/* Computes node keys and values of levels 1..max(J(T), J_keep) over tokens
 * [0, T). Only nodes whose token range reaches past t_from are (re)computed,
 * so t_from = 0 builds everything and t_from = old T refreshes a tree after
 * tokens were added. Knode[j], Vnode[j] (j >= 1) are caller-owned fp64
 * arrays of at least ceil(T / b^j) rows. W is the d x d pooler, row-major,
 * y = W x. Returns the number of levels computed. */
int orc_build(const void* Ktok, const void* Vtok, int tok_dtype, long long T, int d, int b, const float* W,
              int storage, long long t_from, int J_keep, double* const* Knode, double* const* Vnode);

/* Keys of the level above n_children given child keys (fp64 rows, as
 * stored): row m = round(W * mean of children [m b, min((m+1) b, n))).
 * out holds ceil(n_children / b) rows. Returns 0, or -1 on bad arguments. */
int orc_pool_level(const double* child_keys, long long n_children, int d, int b, const float* W, int storage,
                   double* out);

/* One query of one unit (a KV head and its G query heads) against the tree
 * over tokens [0, T) (Knode/Vnode levels 1..J(T)) and the level-0 tokens,
 * followed by nloc local tokens (a prefill chunk's own causal tokens; 0 for
 * decode). q is float32 [G][d].
 * Outputs (each nullable except out):
 *   out    [G][d]   attention output per query head;
 *   sel    [J][k]   selected node ids of level j in row j-1, ascending, -1 pad;
 *   margin [J]      S_(k) - S_(k+1) at level j (HUGE_VAL when none dropped);
 *   rows   [2]      {K rows read, V rows read (= softmax entries)}.
 * Returns J(T), or -1 on bad arguments / allocation failure. */
int orc_query(int d, int b, int k, int G, double rope_base, long long T, const double* const* Knode,
              const double* const* Vnode, const void* Ktok, const void* Vtok, int tok_dtype, const void* Kloc,
              const void* Vloc, long long nloc, const float* q, double* out, int* sel, double* margin,
              long long* rows);

/* Gradients of one decode query (no local tokens) with the selections
 * held fixed: dq [G][d] is overwritten; the gradients with respect to the
 * token keys and values (dKtok, dVtok [T][d], through the entries and the
 * summaries) and the pooler (dW [d][d], row-major like W) are added into
 * the given arrays. dout [G][d] is the output gradient. Storage rounding is
 * taken as the identity. Returns J, or -1. */
int orc_query_grad(int d, int b, int k, int G, double rope_base, long long T, const double* const* Knode,
                   const double* const* Vnode, const void* Ktok, const void* Vtok, int tok_dtype, const float* W,
                   const float* q, const double* dout, double* dq, double* dKtok, double* dVtok, double* dW);

/* The same for a prefill query: the tree over tokens [0, T) (T may be 0)
 * plus the chunk's own causal tokens Kloc, Vloc [nloc][d] (as in orc_query);
 * their gradients are added into dKloc, dVloc [nloc][d]. Returns J, or -1. */
int orc_query_grad_local(int d, int b, int k, int G, double rope_base, long long T, const double* const* Knode,
                         const double* const* Vnode, const void* Ktok, const void* Vtok, int tok_dtype,
                         const void* Kloc, const void* Vloc, long long nloc, const float* W, const float* q,
                         const double* dout, double* dq, double* dKtok, double* dVtok, double* dKloc, double* dVloc,
                         double* dW);

/* LSA-style clustered order of T tokens ("Latent Sparse Attention"
 * abstract: keys clustered hierarchically in a learned latent space, queries
 * scoring the hierarchy of clusters). Reading R20 (see the .c file): level j
 * of the tree over the reordered tokens groups them by the latent coordinate
 * z_j(t) = <Z row j-1, k_t>. Z is float32 [J][d] (J = levels(T, b); rows
 * beyond J unused); perm [T] receives the token index placed at each
 * position. Returns J, or -1 on bad arguments / allocation failure. */
int orc_cluster_order(const void* Ktok, int tok_dtype, long long T, int d, int b, const float* Z, int* perm);

#ifdef __cplusplus
}
#endif
#endif
