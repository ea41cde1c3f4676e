"""KV page-table remap after resampling (oracle side).

Test infrastructure only (see ``oracle/__init__``).

"Faster LLM Inference via Sequential Monte Carlo", section 2 (system
optimisation, KV cache management): when a particle is duplicated, its KV
cache is not copied; only page pointers / page metadata are.  Reading: a pure
gather of page-table rows by ancestor,

    pt_out[b, i, :]  = pt_in[b, a_i, :]
    tok_out[b, i, :] = tok_in[b, a_i, :]          (optional)
    refcnt[p]        = #{ (b, i, s) : pt_out[b, i, s] == p }   (optional)

Page id -1 marks an empty slot: it is copied and not counted.  Any other id
outside [0, num_pages) is copied, not counted, and raises the page error bit.
An ancestor outside [0, N) fills that particle's rows with -1 and raises the
ancestor error bit.  Copy-on-write of a shared, partly filled tail page stays
with the caller, who can read the reference counts.

Parity status: this is the definition itself; pinned by a hand-built example
and the count identity sum(refcnt) = number of valid entries
(tests/test_oracle_pagetable.py).
"""

import numpy as np

from .score import DEV_ANCESTOR_OOB, DEV_PAGE_OOB


def kv_pagetable_remap(pt_in, ancestors, num_pages=None, tok_in=None):
    pt_in = np.asarray(pt_in, dtype=np.int64)
    anc = np.asarray(ancestors, dtype=np.int64)
    B, N, P = pt_in.shape
    err = 0
    pt_out = np.full((B, N, P), -1, dtype=np.int64)
    tok_out = None
    if tok_in is not None:
        tok_in = np.asarray(tok_in, dtype=np.int64)
        tok_out = np.full(tok_in.shape, -1, dtype=np.int64)
    for b in range(B):
        for i in range(N):
            a = int(anc[b, i])
            if not (0 <= a < N):
                err |= DEV_ANCESTOR_OOB
                continue
            pt_out[b, i] = pt_in[b, a]
            if tok_in is not None:
                tok_out[b, i] = tok_in[b, a]
    refcnt = None
    if num_pages is not None:
        refcnt = np.zeros(int(num_pages), dtype=np.int64)
        flat = pt_out.reshape(-1)
        valid = (flat >= 0) & (flat < num_pages)
        bad = (flat != -1) & ~valid
        # entries of out-of-range ancestors are -1 and are not counted
        if bad.any():
            err |= DEV_PAGE_OOB
        np.add.at(refcnt, flat[valid], 1)
    return dict(pt_out=pt_out, tok_out=tok_out, refcnt=refcnt, err=err)
