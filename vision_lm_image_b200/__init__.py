"""B200-native MiMo-V2 image preprocessing.

The pixel path of MimoV2ImageProcessor (smart_resize geometry, RGBA onto
white, bilinear resize on 0..255, mean/std normalisation, T=2 duplication,
merge-block patch rows and the column-order permutation) as a C-ABI library
(``include/mimo.h``) backed by hand-written sm_100a CUDA kernels. This package
is the thin Python binding over that library.
"""
from .mimo import (  # noqa: F401
    BF16, F32, ROW_WIDTH, MimoError, MimoLibraryMissing, MimoParams, PackedBatch, get_number_of_image_patches,
    lib, make_params, pack_images, plan_batch, preprocess, preprocess_batch, preprocess_batch_host,
    smart_resize, smart_resize_status,
)

__version__ = "0.1.0"
