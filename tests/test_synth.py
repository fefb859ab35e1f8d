"""The seeded input generators: shapes, ranges and the surjective map."""
import numpy as np
import torch

from hashed_gram_embedding_compress_b200 import synth


def test_comp_map_is_a_surjection_onto_cvocab():
    for name in ("tiny_f32", "prefill_bf16", "large_hbm"):
        sh = synth.SHAPES[name]
        m = synth.make_comp_map(sh, synth.stream_seeds(sh))
        assert m.shape == (sh.vocab,) and m.dtype == torch.int32
        assert int(m.min()) == 0 and int(m.max()) == sh.cvocab - 1
        assert torch.unique(m).numel() == sh.cvocab


def test_tokens_in_range_and_zipfian():
    sh = synth.SHAPES["prefill_bf16"]
    x = synth.make_tokens(sh, synth.stream_seeds(sh))
    assert x.shape == (sh.B, sh.T) and x.dtype == torch.int32
    assert int(x.min()) >= 0 and int(x.max()) < sh.vocab
    cnt = np.sort(np.bincount(x.reshape(-1).numpy(), minlength=sh.vocab))[::-1]
    # rank-frequency slope in log-log space close to -s for the head of the distribution
    r = np.arange(1, 201)
    slope = np.polyfit(np.log(r), np.log(cnt[:200] + 1e-9), 1)[0]
    assert -1.35 < slope < -0.85


def test_seeded_draws_repeat():
    sh = synth.SHAPES["tiny_f32"]
    s1, s2 = synth.stream_seeds(sh), synth.stream_seeds(sh)
    assert s1 == s2 and len(set(s1.values())) == len(s1)
    assert torch.equal(synth.make_tokens(sh, s1), synth.make_tokens(sh, s2))
    t1 = synth.make_tables([11, 13], 4, "bf16", s1)
    t2 = synth.make_tables([11, 13], 4, "bf16", s2)
    assert all(torch.equal(a, b) for a, b in zip(t1, t2))
    wk, wv, nq, nk = synth.make_weights(sh, s1)
    assert wk.shape == (1, 128, 256) and wv.shape == (128, 256) and nq.shape == (1, 128)
    h = synth.make_hidden(sh, s1)
    assert h.shape == (128, 1, 128) and h.dtype == torch.float32
