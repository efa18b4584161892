"""Test inputs for the warp-staged pixel kernel: batches whose every image shrinks under max_pixels."""
import oracle
import workloads


def shrunk_batch(seed, n, max_pixels, lo=250, hi=520):
    """RGB and RGBA images whose every side shrinks by 1.25 to 1.9 under max_pixels: no axis gathers taps
    and every height shrinks by at least 1.25, so a launch of them takes the warp-staged kernel."""
    rng = workloads.rng_for(seed)
    imgs = []
    while len(imgs) < n:
        h, w = int(rng.integers(lo, hi)), int(rng.integers(lo, hi))
        hr, wr = oracle.smart_resize(h, w, max_pixels=max_pixels)
        if not (4 * h >= 5 * hr and 10 * h <= 19 * hr and 10 * w <= 19 * wr):
            continue
        imgs.append(workloads.rgba_image(rng, h, w) if len(imgs) % 2 else workloads.uniform_image(rng, h, w, 3))
    return imgs
