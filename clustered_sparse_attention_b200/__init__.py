"""B200-native clustered sparse attention (SVG-EAR on SVG2's permutation).

The compute path lives in libsvgear.so (CUDA, sm_100a) behind the C ABI of
include/svgear.h; ``_lib`` is its thin ctypes binding.  Import of the
package does not load the library; the first call does, and raises if the
library is missing -- there is no CPU path.
"""
from ._lib import (Clustering, SvgearError, kernel_launches, layer, layer_host, lib, svgear_attend, svgear_centroids,
                   svgear_cluster, svgear_kmeans_assign, svgear_kmeans_update,
                   svgear_kmeanspp_init, svgear_label_sort, svgear_permute, svgear_probe,
                   svgear_route, svgear_route_select, svgear_route_select_budget,
                   svgear_route_topp, svgear_topp_budget, svgear_key_variance,
                   svgear_probe_value_free, svgear_diagnostics, svgear_layer, workspace_bytes)

__all__ = ["Clustering", "SvgearError", "kernel_launches", "layer", "layer_host", "lib", "svgear_attend", "svgear_centroids",
           "svgear_cluster", "svgear_kmeans_assign", "svgear_kmeans_update",
           "svgear_kmeanspp_init", "svgear_label_sort", "svgear_permute", "svgear_probe",
           "svgear_route", "svgear_route_select", "svgear_route_select_budget",
           "svgear_route_topp", "svgear_topp_budget", "svgear_key_variance",
           "svgear_probe_value_free", "svgear_diagnostics", "svgear_layer", "workspace_bytes"]
