"""Host side of the coordinated noise initialisation (no GPU): the library's frame selection
(dp_coordinated_frames, through the binding) equals the oracle's over a whole long run."""
import oracle as O
from workloads import make_noise_permutations


def test_binding_rule_matches_the_oracle():
    import long_video_diffusion_b200 as dp
    frames = [2] * 128 + [1]
    perms = make_noise_permutations(len(frames), 16, seed=9)
    sched = O.coordinated_schedule(frames, 8, perms)
    got = dp.coordinated_schedule(frames, 8, perms)
    assert got[:8] == [[2 * b, 2 * b + 1] for b in range(8)]
    assert got == sched
