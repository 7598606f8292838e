"""Covering rate of the multiplicative codebook (the pages' Proposition 3.1:
the 24 S codewords q_p q_s of random q_s cover S^3 at a rate
O((24 S)^(-1/3))): a statistical check on the oracle's own search.

For Haar-random unit quaternions u, the angle to the nearest codeword is
arccos of the oracle's best score <u, c>.  Over S = 1 .. 64 the mean angle
falls as (24 S)^slope with the slope near -1/3, the exponent of N points
spread over the 3-dimensional sphere: the fitted slope must lie in
[-0.40, -0.27] and the angles must fall monotonically.  S = 1 is a closed
case: the codewords are the 24 elements of 2T (rotated by one unit q_s),
the vertices of a 24-cell, whose deep holes sit at exactly 45 degrees."""
import numpy as np


def nearest_angles(oracle, S, n, seed):
    rng = np.random.default_rng(seed)
    u = rng.standard_normal((n, 4))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    x = u.astype(np.float32).reshape(1, 1, n // 32, 128)
    cb = oracle.make_codebook(11, S, 1)
    _, _, best, _, _ = oracle.encode(x, cb, S)
    return np.arccos(np.clip(best.astype(np.float64), -1.0, 1.0))


def test_mean_angle_falls_as_the_cube_root_of_the_codebook_size(oracle):
    Ss = [1, 2, 4, 8, 16, 32, 64]
    means, maxes = [], []
    for S in Ss:
        a = nearest_angles(oracle, S, 4096, S)
        means.append(a.mean())
        maxes.append(a.max())
    slope = np.polyfit(np.log(24.0 * np.array(Ss)), np.log(means), 1)[0]
    print("[covering] mean angle (deg) %s, max %s, slope %.3f"
          % (np.round(np.degrees(means), 2), np.round(np.degrees(maxes), 2), slope))
    assert -0.40 <= slope <= -0.27, slope
    assert np.all(np.diff(means) < 0)


def test_2t_alone_covers_within_its_known_radius(oracle):
    """S = 1: the codewords are the 24 elements of 2T times one unit q_s, the
    vertices of a (rotated) 24-cell.  Its deep holes are the vertices of the
    dual 24-cell, e.g. (1, 1, 0, 0)/sqrt(2), at exactly 45 degrees from the
    nearest vertex; no unit quaternion is farther, and a large sample comes
    close to that bound."""
    a = nearest_angles(oracle, 1, 32768, 5)
    assert a.max() <= np.radians(45.0) + 1e-5
    assert a.max() >= np.radians(40.0)             # the sample gets near the deep holes
