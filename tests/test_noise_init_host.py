"""Host side of the coordinated noise initialisation (no GPU): the binding's frame-selection
rule equals the oracle's over a whole long run."""
import oracle as O
from workloads import make_noise_permutations


def test_binding_rule_matches_the_oracle():
    import long_video_diffusion_b200 as dp
    frames = [2] * 128 + [1]
    perms = make_noise_permutations(len(frames), 16, seed=9)
    sched = O.coordinated_schedule(frames, 8, perms)
    got = [[2 * b, 2 * b + 1] for b in range(8)]
    for b in range(8, len(frames)):
        got.append(dp.coordinated_frames(16, frames[b], got[b - 1], perms[b]))
    assert got == sched
