/*
 * Replays an allocator trace through the C ABI alone (no Python in the loop),
 * for tests/test_c_abi.py.
 *
 * Usage: c_abi_trace NUM_BLOCKS BLOCK_SIZE < trace
 * stdin: the initial free order (a line "O n id0 id1 ..."), then one
 * operation per line:
 *   A          add a sequence                     -> "A <seq>"
 *   P <seq>    append one token                   -> "P <slot> <old> <new>" (old = new = -1
 *                                                     without a copy) or "P OOM"
 *   N <seq> k  append k tokens (a prompt)         -> "N <first slot> <last slot> <copies>" or "N OOM"
 *   F <seq>    fork                               -> "F <child>"
 *   X <seq>    free                               -> "X"
 *   R          checkpoint and resume: snapshot the pool and tables, restore
 *              them into new objects, destroy the old ones, carry on with
 *              the restored pair                  -> "R <snapshot bytes>"
 * At the end it prints the pool and every live table:
 *   "RC n c0 c1 ...", "FREE n b0 b1 ...", "T <seq> <len> <nblocks> b0 b1 ..."
 * Exit status 0, or 1 with a message on stderr when a call fails unexpectedly.
 */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "pagedkv.h"

static int check(int rc, const char* what) {
  if (rc != PA_OK) {
    fprintf(stderr, "%s: %s (%s)\n", what, pa_strerror(rc), pa_last_error());
    exit(1);
  }
  return rc;
}

int main(int argc, char** argv) {
  if (argc != 3) {
    fprintf(stderr, "usage: %s NUM_BLOCKS BLOCK_SIZE < trace\n", argv[0]);
    return 1;
  }
  const int nb = atoi(argv[1]), bs = atoi(argv[2]);
  int32_t* order = (int32_t*)malloc(sizeof(int32_t) * (size_t)nb);
  int32_t* buf = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nb + 1));
  int64_t* pairs = (int64_t*)malloc(sizeof(int64_t) * 2 * (size_t)(nb * bs + 1));
  int32_t* slots = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nb * bs + 1));
  if (!order || !buf || !pairs || !slots) return 1;

  char op[8];
  int n = 0;
  if (scanf("%7s %d", op, &n) != 2 || strcmp(op, "O") != 0 || n != nb) {
    fprintf(stderr, "trace must start with the free order\n");
    return 1;
  }
  for (int i = 0; i < nb; ++i)
    if (scanf("%d", &order[i]) != 1) return 1;

  pa_alloc* pool = NULL;
  pa_seqs* seqs = NULL;
  check(pa_alloc_create(nb, order, &pool), "pa_alloc_create");
  check(pa_seqs_create(pool, bs, &seqs), "pa_seqs_create");

  while (scanf("%7s", op) == 1) {
    int32_t sid = 0, out = 0, n_cow = 0, n_done = 0;
    if (strcmp(op, "A") == 0) {
      check(pa_seqs_add(seqs, &out), "pa_seqs_add");
      printf("A %d\n", out);
    } else if (strcmp(op, "P") == 0) {
      if (scanf("%d", &sid) != 1) return 1;
      const int rc = pa_seqs_append(seqs, &sid, 1, slots, pairs, &n_cow, &n_done);
      if (rc == PA_ERR_OOM) {
        printf("P OOM\n");
      } else {
        check(rc, "pa_seqs_append");
        if (n_cow) printf("P %d %lld %lld\n", slots[0], (long long)pairs[0], (long long)pairs[1]);
        else printf("P %d -1 -1\n", slots[0]);
      }
    } else if (strcmp(op, "N") == 0) {
      int k = 0;
      if (scanf("%d %d", &sid, &k) != 2 || k < 1 || k > nb * bs) return 1;
      const int rc = pa_seqs_append_n(seqs, sid, k, slots, pairs, &n_cow);
      if (rc == PA_ERR_OOM) {
        printf("N OOM\n");
      } else {
        check(rc, "pa_seqs_append_n");
        printf("N %d %d %d\n", slots[0], slots[k - 1], n_cow);
      }
    } else if (strcmp(op, "F") == 0) {
      if (scanf("%d", &sid) != 1) return 1;
      check(pa_seqs_fork(seqs, sid, &out), "pa_seqs_fork");
      printf("F %d\n", out);
    } else if (strcmp(op, "R") == 0) {
      uint64_t bytes = 0;
      check(pa_seqs_snapshot(seqs, NULL, 0, &bytes), "pa_seqs_snapshot size");
      void* snap = malloc(bytes ? bytes : 1);
      if (!snap) return 1;
      check(pa_seqs_snapshot(seqs, snap, bytes, &bytes), "pa_seqs_snapshot");
      pa_alloc* pool2 = NULL;
      pa_seqs* seqs2 = NULL;
      check(pa_seqs_restore(snap, bytes, &pool2, &seqs2), "pa_seqs_restore");
      free(snap);
      check(pa_seqs_destroy(seqs), "pa_seqs_destroy");
      check(pa_alloc_destroy(pool), "pa_alloc_destroy");
      pool = pool2;
      seqs = seqs2;
      printf("R %llu\n", (unsigned long long)bytes);
    } else if (strcmp(op, "X") == 0) {
      if (scanf("%d", &sid) != 1) return 1;
      check(pa_seqs_free(seqs, sid), "pa_seqs_free");
      printf("X\n");
    } else {
      fprintf(stderr, "unknown operation %s\n", op);
      return 1;
    }
  }

  check(pa_alloc_refcounts(pool, buf, nb), "pa_alloc_refcounts");
  printf("RC %d", nb);
  for (int i = 0; i < nb; ++i) printf(" %d", buf[i]);
  printf("\n");
  int32_t nfree = 0;
  check(pa_alloc_free_list(pool, buf, nb, &nfree), "pa_alloc_free_list");
  printf("FREE %d", nfree);
  for (int i = 0; i < nfree; ++i) printf(" %d", buf[i]);
  printf("\n");

  int32_t nlive = 0;
  check(pa_seqs_live(seqs, NULL, 0, &nlive), "pa_seqs_live");
  int32_t* live = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nlive + 1));
  check(pa_seqs_live(seqs, live, nlive, &nlive), "pa_seqs_live");
  for (int i = 0; i < nlive; ++i) {
    int32_t len = 0, nblk = 0;
    check(pa_seqs_len(seqs, live[i], &len), "pa_seqs_len");
    check(pa_seqs_table(seqs, live[i], buf, nb, &nblk), "pa_seqs_table");
    printf("T %d %d %d", live[i], len, nblk);
    for (int j = 0; j < nblk; ++j) printf(" %d", buf[j]);
    printf("\n");
  }
  check(pa_seqs_destroy(seqs), "pa_seqs_destroy");
  check(pa_alloc_destroy(pool), "pa_alloc_destroy");
  free(live);
  free(order);
  free(buf);
  free(pairs);
  free(slots);
  return 0;
}
