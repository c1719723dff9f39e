"""The five synthetic workloads the step is tested and measured on.

Sizes only; no arithmetic of the method lives here.

  toy          4 ranks own blocks A, B, C, D of 65,536 parameters.
  gpt2_small   GPT-2-small-shaped flat vector, stage 2, Nd = 8: 12 blocks of
               (12 h^2 + 13 h) with h = 768 (3072-wide MLP), 50257 x 768 token
               table, 1024 x 768 position table, final norm (2 h):
               124,439,808 parameters.
  stage3_1p3b  stage 3, Nd = 16, layer-wise units of a 24-layer, hidden-2048
               model: token + position tables (50257 + 2048) x 2048, 24 blocks
               of (12 h^2 + 13 h), final norm 2 h: 1,315,723,264 parameters;
               1 % of the gradient entries scaled by 100.
  owner_7p5b   one owner's view of a 7.5B-parameter model at Nd = 64
               (S = 117,187,520 after padding), 25M-element buckets.
  sweep        5e8 parameters, Nd in {2, 4, 8, 16, 64}, buckets of 1 MB ..
               512 MB of one rank's bf16 gradient (bucket_elems = MB * 2^19).
seed_id enters the seeds of the input generators.
"""

ADAM = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8)


def gpt2_small_psi(h=768, layers=12, vocab=50257, positions=1024):
    return layers * (12 * h * h + 13 * h) + vocab * h + positions * h + 2 * h


def stage3_units(h=2048, layers=24, vocab=50257, positions=2048):
    return [(vocab + positions) * h] + [12 * h * h + 13 * h] * layers + [2 * h]


CONFIGS = {
    "toy": dict(seed_id=1, psi=65_536, nd=4, stage=2, bucket_elems=16_384, units=None,
               sigma=0.01, outlier_frac=0.0, steps=3, owner_view=-1,
               workload="toy 4-rank A/B/C/D, psi=65536, Nd=4"),
    "gpt2_small": dict(seed_id=2, psi=gpt2_small_psi(), nd=8, stage=2, bucket_elems=25_000_000, units=None,
               sigma=1e-3, outlier_frac=0.0, steps=10, owner_view=-1,
               workload="GPT-2-small flat vector, psi=124439808, Nd=8, stage 2, 25M-element buckets"),
    "stage3_1p3b": dict(seed_id=3, psi=sum(stage3_units()), nd=16, stage=3, bucket_elems=1 << 27,
               units=stage3_units(), sigma=1e-3, outlier_frac=0.01, steps=5, owner_view=-1,
               workload="stage 3 layer-wise, 24 x hidden 2048 (psi=1315723264), Nd=16"),
    "owner_7p5b": dict(seed_id=4, psi=7_500_000_000, nd=64, stage=2, bucket_elems=25_000_000, units=None,
               sigma=1e-3, outlier_frac=0.0, steps=3, owner_view=0,
               workload="one owner of a 7.5B model at Nd=64 (S=117187520), 25M buckets"),
}


def sweep_config(nd, bucket_mb):
    return dict(seed_id=5, psi=500_000_000, nd=nd, stage=2, bucket_elems=bucket_mb << 19, units=None,
                sigma=1e-3, outlier_frac=0.0, steps=3, owner_view=-1,
                workload="bucket sweep psi=5e8, Nd=%d, %d MB buckets" % (nd, bucket_mb))
