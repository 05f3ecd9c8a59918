"""Every buffer the library writes sits between canary regions; after a full eviction
the canaries must be intact (device-side out-of-bounds writes show up here, without a
sanitizer)."""
import numpy as np
import pytest
import torch

import synth
from tests.parity_utils import to_dev

pytestmark = pytest.mark.gpu

CANARY = 0x7F7F7F7F
PAD = 64 * 1024  # bytes of canary before and after each buffer


class Arena:
    """One int32 allocation carved into buffers separated by canary pads."""

    def __init__(self, sizes):
        self.offsets = {}
        off = PAD
        for name, nbytes in sizes.items():
            self.offsets[name] = (off, nbytes)
            off += (nbytes + 255) // 256 * 256 + PAD
        self.raw = torch.full((off // 4,), CANARY, dtype=torch.int32, device="cuda")

    def view(self, name, dtype, shape):
        off, nbytes = self.offsets[name]
        words = self.raw[off // 4: (off + nbytes + 3) // 4]
        return words.view(torch.uint8)[:nbytes].view(dtype).view(shape)

    def ptr(self, name):
        return self.raw.data_ptr() + self.offsets[name][0]

    def check(self):
        host = self.raw.cpu().numpy()
        keep = np.ones(host.size, dtype=bool)
        for off, nbytes in self.offsets.values():
            keep[off // 4: (off + nbytes + 3) // 4] = False
        bad = np.nonzero(keep & (host != CANARY))[0]
        assert bad.size == 0, f"{bad.size} canary words overwritten, first at byte {bad[0] * 4}"


# shapes beyond the named workloads: one 256-column TMEM stage per group, split tiles at
# d = 64, and long head-aligned runs
EXTRA = {
    "wide_stage_g8": synth.small("llama8b_32k", hq=8, hkv=1, seq_len=1100, window=32, budget=200),
    "split_d64": synth.small("tiny", hq=6, hkv=1, seq_len=900, window=48, budget=200),
    "long_128k_b10": synth.WORKLOADS["long_128k_b10"],
}


@pytest.mark.parametrize("name,budget", [("tiny", None), ("llama8b_32k", None), ("llama8b_32k", 128),
                                         ("gqa7_batched", None), ("wide_stage_g8", None),
                                         ("split_d64", None), ("long_128k_b10", None)])
def test_no_write_outside_buffers(name, budget):
    import token_eviction_b200 as m
    wl = EXTRA.get(name) or synth.WORKLOADS[name]
    B = wl.budget if budget is None else budget
    b, hq, hkv, d, L, w = wl.batch, wl.hq, wl.hkv, wl.head_dim, wl.seq_len, wl.window
    sh = m.make_shape(b, hq, hkv, d, L, w, B)
    inp = synth.make_inputs(wl)
    q, k, v = to_dev(inp.q_win), to_dev(inp.k), to_dev(inp.v)
    ws = m.kvp_workspace_bytes(sh)
    ar = Arena({"ws": ws, "score": b * hkv * L * 4, "s1": b * hkv * L * 4, "s2": b * hkv * L * 4,
                "idx": b * hkv * B * 4, "k_out": b * hkv * B * d * 2, "v_out": b * hkv * B * d * 2})
    score = ar.view("score", torch.float32, (b, hkv, L))
    s1 = ar.view("s1", torch.float32, (b, hkv, L))
    s2 = ar.view("s2", torch.float32, (b, hkv, L))
    idx = ar.view("idx", torch.int32, (b, hkv, B))
    ko = ar.view("k_out", torch.bfloat16, (b, hkv, B, d))
    vo = ar.view("v_out", torch.bfloat16, (b, hkv, B, d))
    wsv = ar.view("ws", torch.uint8, (ws,))
    for _ in range(2):
        m.kvp_score(sh, q, k, v, score, s1, s2, wsv)
        m.kvp_select(sh, score, idx, wsv)
        m.kvp_compact(sh, k, v, idx, ko, vo)
    torch.cuda.synchronize()
    ar.check()
