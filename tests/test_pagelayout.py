"""The numpy page reader used by the GPU tests covers every byte of a page exactly
once (no field overlaps another, none is left out)."""
import pytest

from tests import pagelayout


@pytest.mark.parametrize("D", [128, 256])
def test_page_fields_partition_the_page(D):
    pagelayout.check_maps_are_permutations(D)
    assert pagelayout.page_bytes(D) == 2 * pagelayout.rec_bytes(D)
