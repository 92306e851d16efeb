"""moe_permute_noalloc — the permute for callers that cannot allocate device
memory (for example an engine step that has reserved all of HBM and forbids
allocation mid-step, or a custom-op host that hands over only input and output
tensors).  It must give exactly what moe_permute gives with a caller-provided
workspace, on two calls in a row (the second call reuses the library's
scratch array, which still holds the first call's contents).

This file is collected last so that a run stopping at the first failure has
already run every other test."""
import numpy as np
import pytest
import torch

from _util import dev, host, rand_bf16, same_bits

pytestmark = pytest.mark.gpu


def _case(rng, T, E, k, zipf):
    p = np.arange(1, E + 1, dtype=np.float64) ** -zipf
    p /= p.sum()
    keys = np.log(p)[None, :] - np.log(-np.log(rng.random((T, E))))
    return np.argsort(-keys, axis=1, kind="stable")[:, :k].astype(np.int32)


# (T, E, k, D, zipf, align), in call order: each smaller problem follows a
# larger one, so a call finds the array holding a bigger call's contents.  The
# first and third have more than 64 chunks of routed entries, which runs the
# separate count, scan and place passes (block bases written by one kernel
# into the array and read by the next); the others run the fused place pass.
CASES = [(16384, 32, 8, 256, 1.2, 128), (4096, 64, 6, 512, 1.1, 128), (20000, 16, 4, 128, 0.0, 1),
         (3000, 32, 8, 256, 0.5, 1)]


def test_permute_noalloc_matches_permute_and_oracle(orc):
    from oracle import layer as OL
    from moe_expert_layer_replay_b200 import abi, build
    build.build()
    A = abi
    for call, (T, E, k, D, zipf, align) in enumerate(CASES):
        rng = np.random.default_rng(40 + call)
        idx = _case(rng, T, E, k, zipf)
        x = rand_bf16(rng, (T, D))
        d = A.dims(T, D, 128, E, k, align)
        R = A.rows_capacity(d)
        outs = []
        for noalloc in (False, True):
            g = lambda *s, dt=torch.int32: torch.full(s, -7, dtype=dt, device="cuda") if dt == torch.int32 \
                else torch.zeros(*s, dtype=dt, device="cuda")
            counts, offsets, pos, src = g(E), g(E + 1), g(T, k), g(R)
            xq, xs = g(R, D, dt=torch.uint8), g(D // 128, R, dt=torch.float32)
            if noalloc:
                A.permute_noalloc(dev(idx), d, counts, offsets, pos, src, dev(x), xq, xs)
            else:
                ws = torch.empty(A.permute_workspace_size(d), dtype=torch.uint8, device="cuda")
                A.permute(dev(idx), d, counts, offsets, pos, src, dev(x), xq, xs, None, None, ws)
            torch.cuda.synchronize()
            Rp = int(host(offsets)[E])
            outs.append([host(counts), host(offsets), host(pos), host(src), host(xq)[:Rp], host(xs)[:, :Rp]])
        for a, b, name in zip(outs[0], outs[1], ["counts", "offsets", "pos", "src_idx", "xq", "xs"]):
            same_bits(b, a, f"call {call}: {name} (no-alloc vs workspace)")
        # and both against the oracle
        oc, oo, op, osrc = orc.permute(idx, E, align, R)
        for got, ref, name in zip(outs[1][:4], [oc, oo, op, osrc], ["counts", "offsets", "pos", "src_idx"]):
            same_bits(got, ref, f"call {call}: {name} (oracle)")
        Rp = int(oo[E])
        q_ref, s_ref = orc.quant_block(OL.dispatch_rows(x, osrc, np.arange(Rp), k), 1, 128)
        same_bits(outs[1][4], q_ref, f"call {call}: xq (oracle)")
        same_bits(outs[1][5].T, s_ref, f"call {call}: xs (oracle)")


def test_permute_noalloc_rejects_oversize():
    from moe_expert_layer_replay_b200 import abi
    d = abi.dims(600000, 128, 128, 256, 8, 128)   # workspace > 1 MiB
    g = lambda *s: torch.empty(*s, dtype=torch.int32, device="cuda")
    with pytest.raises(abi.MoeError) as e:
        abi.permute_noalloc(g(8), d, g(256), g(257), g(8), g(8), None, None, None)
    assert e.value.status == abi.UNSUPPORTED
