"""Prints the grouping error table of the design notes (CPU only):
``python -m tests.diag_table``.  It draws the seeded synthetic workloads with
``synth`` and measures them with ``oracle.diag``."""
import numpy as np

from bit_asymmetric_kv_prefill_b200 import synth
from oracle.diag import MODES, errors


def table(T: int = 1024, heads: int = 4, queries: int = 8):
    """Rows (workload, rope, mode, errors) of the error table on the seeded
    synthetic workloads: T tokens (256 for tiny), `heads` kv heads (2 for tiny)
    of batch element 0, `queries` decode queries per head; key_rel and
    value_rel divide the errors by the mean per-head Frobenius norm.
    ``python -m tests.diag_table`` prints it as markdown."""
    rows = []
    for name, rope in (("tiny", None), ("llama2_7b_layer", None), ("llama2_13b_cache", None),
                       ("long_context", "pre"), ("long_context", "post")):
        tiny = name == "tiny"
        w = synth.scaled(synth.WORKLOADS[name], B=1, H_kv=2 if tiny else heads,
                         H_q=2 if tiny else heads, T=256 if tiny else T)
        K, V = synth.prefill_inputs(w, seed=0)
        K, V = K.float().numpy()[0], V.float().numpy()[0]
        q = np.stack([synth.step_inputs(w, s)[2].float().numpy()[0] for s in range(queries)], 1)
        nk = float(np.mean([np.linalg.norm(k) for k in K.astype(np.float64)]))
        nv = float(np.mean([np.linalg.norm(v) for v in V.astype(np.float64)]))
        for mode in MODES:
            e = errors(K, V, q, mode, rope=rope)
            e.update(key_rel=e["key"] / nk, value_rel=e["value"] / nv)
            rows.append((name, rope, mode, e))
    return rows


def main():
    print("| workload | keys | grouping | key error | value error | attention-output error % |")
    print("|---|---|---|---|---|---|")
    for name, rope, mode, e in table():
        keys = {None: "", "pre": "pre-RoPE", "post": "post-RoPE"}[rope]
        print(f"| {name} | {keys} | {mode} | {e['key']:.1f} ({e['key_rel']:.3f}) | "
              f"{e['value']:.1f} ({e['value_rel']:.3f}) | {e['attn']:.1f} |")


if __name__ == "__main__":
    main()
