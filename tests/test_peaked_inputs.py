"""The peaked inputs of the GPU parity tests, checked on the host.

They must reach the code they are meant for -- tiles whose maximum is more
than 8 (base 2) above the running maximum, where the prefill kernel rescales O
in tensor memory -- and the oracle must give the closed forms they imply: the
mean of V for equal scores, the value row of a key ~950 (base 2) above the
rest.
"""

import numpy as np
import torch

import peaked as PK
from oracle import attention as OA
from paged_kv_cache_364_b200 import synthetic as syn

PREFILL_CASES = [(1, 1), (64, 64), (65, 65), (300, 300), (700, 200), (1000, 37), (129, 129), (17, 5),
                 (450, 450)]


def test_inputs_reach_the_tensor_memory_rescale():
    """Rows of the prefill cases see tiles after the first whose maximum is
    more than 8 above the running maximum (rising, staircase, near-threshold
    columns), and none for falling or flat scores."""
    w = syn.custom_prefill(*zip(*PREFILL_CASES), 32, 8, 128, "bf16", seed=350)
    vals = PK.column_values(w.lens, w.scale, w.torch_dtype, 351, int(w.lens.max())).numpy()
    grows = {name: 0 for name in PK.PATTERNS}
    for s, (n, q) in enumerate(zip(w.lens, w.qlens)):
        for pos in range(int(n - q), int(n)):
            for c, name in enumerate(PK.PATTERNS):
                grows[name] += PK.tiles_that_grow(vals[s], w.scale, pos + 1, c)
    assert grows["rise"] > 1000 and grows["steps"] > 100 and grows["near_threshold"] > 100
    assert grows["fall"] == 0 and grows["flat"] == 0


def test_scores_are_exact_and_within_the_cap():
    """The stored K values times QV are the kernels' scores: exact in fp32
    (one non-zero product), and |scaled score| < 2^10."""
    for dtype in (torch.bfloat16, torch.float16):
        w = syn.custom_workload([1, 70, 3000], 32, 8, 128, "bf16", seed=1)
        vals = PK.column_values(w.lens, w.scale, dtype, 2, 3008)
        prod32 = (vals * PK.QV).to(torch.float32)
        assert torch.equal(prod32.double(), vals.double() * PK.QV)
        assert PK.score_max(vals, w.scale) < 1024


def test_oracle_closed_forms_on_peaked_inputs():
    w = syn.custom_workload([1, 5, 100, 700], 8, 4, 64, "bf16", seed=3)
    inp = syn.decode_inputs(w, "cpu")
    tables = inp.block_tables.numpy()
    vals = PK.column_values(w.lens, w.scale, w.torch_dtype, 4, tables.shape[1] * 16)
    PK.fill_cache(inp.k_cache, tables, w.lens, vals)
    PK.set_queries(inp.q, 2)
    ref = OA.paged_decode(inp.q, inp.k_cache, inp.v_cache, inp.block_tables, inp.context_lens, w.scale)
    V = [OA.gather_sequence(inp.v_cache.double().numpy(), tables[s], int(n), hk)
         for s, n in enumerate(w.lens) for hk in range(4)]
    col = {name: c for c, name in enumerate(PK.PATTERNS)}
    checked = 0
    for s, n in enumerate(w.lens):
        n = int(n)
        for h in range(8):
            hk = h // 2
            v = V[s * 4 + hk]
            c = PK.pattern_column(h, 2)
            if c == col["flat"]:
                np.testing.assert_allclose(ref[s, h], v.mean(0), atol=1e-12)
                checked += 1
            elif c == col["last_key"]:
                np.testing.assert_allclose(ref[s, h], v[n - 1], atol=1e-12)
                checked += 1
            elif c == col["dominant_mid"]:
                np.testing.assert_allclose(ref[s, h], v[n // 3], atol=1e-12)
                checked += 1
    assert checked >= 3 * 3
