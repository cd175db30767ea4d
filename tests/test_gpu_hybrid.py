"""GPU parity of the hybrid cache (BF16 sink and recent window, quantized history).

Policy (a reading; the pages fix no sizes): the sink is the first k tokens, k a
whole number of pages; the history grows a page at a time, so it holds
64 * floor((T - k - w) / 64) tokens once T > k + w, and the window keeps the
remaining newest w .. w + 63 tokens. The oracle derives both segments from this
definition and the token values alone; the GPU side follows the same policy
with its own page bookkeeping (append into the window, move whole pages).
"""
import numpy as np
import pytest
import torch

from bit_mla_kv_qdecode_b200 import api, synth
from oracle import attention, layout
from tests import mla_cases as mc

pytestmark = pytest.mark.gpu

PAGE = 64


def hist_len(T, k, w):
    return max(0, (T - k - w) // PAGE * PAGE)


def tokens_f32(w, B, T, mag):
    """Token values (bf16-exact float32) [B, T, 576] from the seeded generator."""
    return np.stack([synth.bf16_bits_to_f32(synth.cache_tokens_bf16(w, b, T, mag)) for b in range(B)])


def oracle_hybrid(desc, x, lens, k, win, qc, qr, scale):
    """Oracle result from the policy definition: pack the history with the
    oracle packer, copy the protected tokens into a float BF16-pool image."""
    B = len(lens)
    maxp = max(1, max((int(T) + PAGE - 1) // PAGE for T in lens))
    pool = layout.new_pool(desc, B * maxp)
    table = np.arange(B * maxp).reshape(B, maxp)
    prot_pool = np.zeros((B * maxp, PAGE, 576), np.float32)
    hl, pl = [], []
    for b, T in enumerate(lens):
        h = hist_len(int(T), k, win)
        if h:
            layout.append(desc, pool, table[b:b + 1], [0], x[b:b + 1, k:k + h, :512], x[b:b + 1, k:k + h, 512:])
        prot = np.concatenate([x[b, :min(k, T)], x[b, k + h:T]])
        for j in range(len(prot)):
            prot_pool[table[b][j // PAGE], j % PAGE] = prot[j]
        hl.append(h)
        pl.append(len(prot))
    return attention.hybrid_decode(desc, pool, table, hl, prot_pool, table, pl, qc, qr, scale)


def test_page_move_packs_like_the_oracle():
    w = synth.workload(1).scaled(B=3)
    desc_o = layout.Desc()
    x = tokens_f32(w, 3, 2 * PAGE, synth.channel_magnitudes(w))
    bits = synth.f32_to_bf16_bits(x)
    bpool = api.new_bf16_pool(6)
    bview = bpool.view(torch.int16).view(6, PAGE, 576)
    src = [4, -1, 1]  # request 1 moves nothing
    for b in range(3):
        bview[src[b] if src[b] >= 0 else 5].copy_(torch.from_numpy(bits[b, PAGE:].view(np.int16)))
    desc = api.make_desc(4, 64, 4, 64, num_pages=6)
    qpool = api.new_qcache_pool(desc)
    table = torch.tensor([[0, 1], [2, 3], [4, 5]], dtype=torch.int32, device="cuda")
    lens_before = torch.tensor([64, 0, 0], dtype=torch.int32, device="cuda")
    api.mla_qcache_append_bf16_pages(desc, qpool, table, lens_before, bpool,
                                     torch.tensor(src, dtype=torch.int32, device="cuda"))
    assert api.mla_get_device_status() == 0
    ref = layout.new_pool(desc_o, 6)
    tab = table.cpu().numpy()
    for b, pos in ((0, 64), (2, 0)):
        layout.append(desc_o, ref, tab[b:b + 1], [pos], x[b:b + 1, PAGE:, :512], x[b:b + 1, PAGE:, 512:])
    assert np.array_equal(qpool.cpu().numpy(), ref), "moved pages differ from the oracle's packing"


class GpuHybrid:
    """Device side of the policy: BF16 pages for the sink and window (position
    order), quantized pages for the history, host-side page bookkeeping."""

    def __init__(self, desc_bits, B, k, win, max_tokens):
        self.B, self.k, self.win = B, k, win
        self.maxp = (max_tokens + PAGE - 1) // PAGE + 2
        self.desc = api.make_desc(*desc_bits, num_pages=B * self.maxp)
        self.qpool = api.new_qcache_pool(self.desc)
        self.bpool = api.new_bf16_pool(B * self.maxp)
        self.q_pages = [[] for _ in range(B)]
        self.p_pages = [[] for _ in range(B)]
        self.free_q = list(range(B * self.maxp))[::-1]
        self.free_b = list(range(B * self.maxp))[::-1]
        self.hist = [0] * B
        self.prot = [0] * B

    def _table(self, pages):
        t = np.full((self.B, self.maxp), 0, np.int32)
        for b, p in enumerate(pages):
            t[b, :len(p)] = p
        return torch.from_numpy(t).cuda()

    def append(self, x_new):
        """x_new float32 [B, n, 576]: into the window, then move full pages out."""
        n = x_new.shape[1]
        for b in range(self.B):
            while len(self.p_pages[b]) * PAGE < self.prot[b] + n:
                self.p_pages[b].append(self.free_b.pop())
        bits = torch.from_numpy(synth.f32_to_bf16_bits(x_new).view(np.int16)).cuda().view(torch.bfloat16)
        api.mla_bf16cache_append(self.bpool, self._table(self.p_pages),
                                 torch.tensor(self.prot, dtype=torch.int32, device="cuda"),
                                 bits[..., :512].contiguous(), bits[..., 512:].contiguous())
        self.prot = [p + n for p in self.prot]
        while True:
            src = [-1] * self.B
            for b in range(self.B):
                if self.prot[b] - self.k >= self.win + PAGE:
                    src[b] = self.p_pages[b][self.k // PAGE]
                    if len(self.q_pages[b]) * PAGE < self.hist[b] + PAGE:
                        self.q_pages[b].append(self.free_q.pop())
            if all(s < 0 for s in src):
                break
            api.mla_qcache_append_bf16_pages(self.desc, self.qpool, self._table(self.q_pages),
                                             torch.tensor(self.hist, dtype=torch.int32, device="cuda"),
                                             self.bpool, torch.tensor(src, dtype=torch.int32, device="cuda"))
            for b in range(self.B):
                if src[b] >= 0:
                    self.free_b.append(self.p_pages[b].pop(self.k // PAGE))
                    self.hist[b] += PAGE
                    self.prot[b] -= PAGE

    def decode(self, qc, qr, scale, out_dtype=torch.float32):
        B, s_q, H = qc.shape[:3]
        lse = torch.empty((B, s_q, H), dtype=torch.float32, device="cuda")
        out, _ = api.mla_qdecode_hybrid(
            self.desc, self.qpool, self._table(self.q_pages), torch.tensor(self.hist, dtype=torch.int32, device="cuda"),
            max(self.hist), self.bpool, self._table(self.p_pages), torch.tensor(self.prot, dtype=torch.int32, device="cuda"),
            max(self.prot), qc, qr, scale, out_dtype=out_dtype, lse=lse)
        torch.cuda.synchronize()
        return out, lse


def check(out, lse, ref, bf16_out=False):
    o_ref, l_ref = ref
    refd = {b: (o_ref[b], l_ref[b]) for b in range(o_ref.shape[0])}
    err, lerr = mc.parity(out, lse, refd, bf16_out=bf16_out)
    assert err <= mc.RTOL_RMS, f"max err {err:.3e} x RMS"
    assert lerr <= mc.LSE_ATOL, f"lse err {lerr:.3e}"


GRID = [
    # (H, s_q, k, window, lens): the warp-level kernel (16 rows) and the cluster kernel (128+ rows)
    (16, 1, 64, 64, [100, 1000, 64]),
    (8, 2, 64, 128, [400, 130, 1]),
    (128, 1, 64, 64, [700, 257]),
    (128, 2, 128, 96, [640, 200]),
]


@pytest.mark.parametrize("spec", GRID)
def test_hybrid_decode_matches_oracle(spec):
    H, s_q, k, win, lens = spec
    B = len(lens)
    w = synth.workload(2).scaled(B=B, H=H, s_q=s_q, bits_c=4, group_c=64, bits_r=4, group_r=64)
    x = tokens_f32(w, B, max(lens), synth.channel_magnitudes(w))
    g = GpuHybrid((4, 64, 4, 64), B, k, win, max(lens))
    # build each request to its length, one token block at a time (ragged lengths: one request per call)
    for T0 in range(0, max(lens), 97):
        T1 = min(T0 + 97, max(lens))
        for b in range(B):
            lo, hi = min(T0, lens[b]), min(T1, lens[b])
            if hi <= lo:
                continue
            sub = GpuHybrid.__new__(GpuHybrid)  # view of request b
            sub.__dict__.update(g.__dict__)
            sub.B = 1
            sub.q_pages, sub.p_pages = [g.q_pages[b]], [g.p_pages[b]]
            sub.hist, sub.prot = [g.hist[b]], [g.prot[b]]
            sub.append(x[b:b + 1, lo:hi])
            g.hist[b], g.prot[b] = sub.hist[0], sub.prot[0]
    assert api.mla_get_device_status() == 0
    assert g.hist == [hist_len(T, k, win) for T in lens]
    qc_bits, qr_bits = synth.queries_bf16(w)
    qc, qr = mc.bits_to_torch(qc_bits), mc.bits_to_torch(qr_bits)
    out, lse = g.decode(qc, qr, w.scale)
    assert api.mla_get_device_status() == 0
    ref = oracle_hybrid(layout.Desc(), x, lens, k, win, synth.bf16_bits_to_f32(qc_bits),
                        synth.bf16_bits_to_f32(qr_bits), w.scale)
    check(out, lse, ref)


@pytest.mark.parametrize("H", [16, 128])
def test_hybrid_serving_loop(H):
    # append 2 tokens per step (as for two speculative queries), move pages out
    # of the window as they fill, and decode every 8 steps and right after a move
    B, s_q, k, win = 2, 2, 64, 64
    w = synth.workload(4).scaled(B=B, H=H, s_q=s_q, bits_c=4, group_c=64, bits_r=4, group_r=64)
    T0, steps = [90, 150], 70
    x = tokens_f32(w, B, max(T0) + 2 * steps, synth.channel_magnitudes(w))
    g = GpuHybrid((4, 64, 4, 64), B, k, win, max(T0) + 2 * steps)
    for b in range(B):  # initial contexts, one request at a time
        sub = GpuHybrid.__new__(GpuHybrid)
        sub.__dict__.update(g.__dict__)
        sub.B, sub.q_pages, sub.p_pages, sub.hist, sub.prot = 1, [g.q_pages[b]], [g.p_pages[b]], [0], [0]
        sub.append(x[b:b + 1, :T0[b]])
        g.hist[b], g.prot[b] = sub.hist[0], sub.prot[0]
    qc_bits, qr_bits = synth.queries_bf16(w)
    qc, qr = mc.bits_to_torch(qc_bits), mc.bits_to_torch(qr_bits)
    qcf, qrf = synth.bf16_bits_to_f32(qc_bits), synth.bf16_bits_to_f32(qr_bits)
    T = list(T0)
    checked = 0
    for step in range(steps):
        before = list(g.hist)
        g.append(np.stack([x[b, T[b]:T[b] + 2] for b in range(B)]))
        T = [t + 2 for t in T]
        assert g.hist == [hist_len(t, k, win) for t in T]
        if step % 8 == 7 or g.hist != before:
            out, lse = g.decode(qc, qr, w.scale)
            assert api.mla_get_device_status() == 0
            check(out, lse, oracle_hybrid(layout.Desc(), x, T, k, win, qcf, qrf, w.scale))
            checked += 1
    assert checked >= 8 and max(g.hist) >= 2 * PAGE


def test_hybrid_workspace_errors():
    w = synth.workload(1).scaled(B=1, H=16)
    g = GpuHybrid((4, 64, 4, 64), 1, 64, 64, 256)
    x = tokens_f32(w, 1, 256, synth.channel_magnitudes(w))
    g.append(x)
    qc_bits, qr_bits = synth.queries_bf16(w)
    qc, qr = mc.bits_to_torch(qc_bits), mc.bits_to_torch(qr_bits)
    need = api.mla_qdecode_hybrid_workspace_bytes(1, 1, 16, max(g.hist), max(g.prot))
    short = torch.empty(max(need - 256, 256), dtype=torch.uint8, device="cuda")
    with pytest.raises(api.MlaError):
        api.mla_qdecode_hybrid(g.desc, g.qpool, g._table(g.q_pages), torch.tensor(g.hist, dtype=torch.int32,
                               device="cuda"), max(g.hist), g.bpool, g._table(g.p_pages),
                               torch.tensor(g.prot, dtype=torch.int32, device="cuda"), max(g.prot), qc, qr, w.scale,
                               workspace=short)
